// Kernel translation unit: every device kernel of the library and the host
// launchers that build their TMA descriptors and grids.  One translation unit
// so the device error word is a single object per device.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cstring>
#include <mutex>
#include <utility>

#include "skv_internal.h"
#include "skv_device.cuh"

#include "merge_state.cuh"
#include "decode.cuh"
#include "quant.cuh"
#include "prefill.cuh"
#include "smooth.cuh"

namespace skv {

int read_and_clear_device_error(int* code) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return e;
  int v = 0;
  e = cudaMemcpyFromSymbol(&v, g_skv_device_error, sizeof(int));
  if (e != cudaSuccess) return e;
  const int zero = 0;
  e = cudaMemcpyToSymbol(g_skv_device_error, &zero, sizeof(int));
  if (e != cudaSuccess) return e;
  *code = v;
  return 0;
}

namespace {
std::atomic<uint64_t> g_launches{0};
// returns e unchanged; counts n launches when e reports success
int counted(int e, int n) {
  if (e == 0) g_launches.fetch_add(static_cast<uint64_t>(n), std::memory_order_relaxed);
  return e;
}
}  // namespace

void count_launches(int n) { g_launches.fetch_add(static_cast<uint64_t>(n), std::memory_order_relaxed); }
uint64_t launch_count() { return g_launches.load(std::memory_order_relaxed); }

// ------------------------------------------------------------ device info

namespace {
constexpr int kMaxDevices = 64;
std::atomic<int> g_sms[kMaxDevices];  // SM count per device, 0 until first queried
std::mutex g_mu;

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int get_encoder(PFN_cuTensorMapEncodeTiled_v12000* out) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_encode == nullptr) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess) return e;
    if (q != cudaDriverEntryPointSuccess || fn == nullptr) return cudaErrorNotSupported;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  *out = g_encode;
  return 0;
}

CUtensorMapDataType tmap_type(skv_dtype dt) {
  return dt == SKV_FP16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
}

// Tiled map over a 16-bit tensor of `rank` dims (dims[0] innermost, strides in
// bytes for dims 1..rank-1), box {64, box1, ...}, 128-byte swizzle, zero fill.
int make_tmap_ty(CUtensorMap* m, CUtensorMapDataType ty, int rank, const void* base, const uint64_t* dims,
                 const uint64_t* strides_bytes, const uint32_t* box) {
  PFN_cuTensorMapEncodeTiled_v12000 enc;
  int e = get_encoder(&enc);
  if (e) return e;
  cuuint64_t gdim[5];
  cuuint64_t gstr[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    gdim[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
  }
  for (int i = 0; i + 1 < rank; ++i) gstr[i] = strides_bytes[i];
  CUresult r = enc(m, ty, static_cast<cuuint32_t>(rank), const_cast<void*>(base), gdim, gstr, bx, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : static_cast<int>(cudaErrorInvalidValue);
}

int make_tmap(CUtensorMap* m, skv_dtype dt, int rank, const void* base, const uint64_t* dims,
              const uint64_t* strides_bytes, const uint32_t* box) {
  return make_tmap_ty(m, tmap_type(dt), rank, base, dims, strides_bytes, box);
}
}  // namespace

int sm_count() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0) return 0;
  if (dev < kMaxDevices) {
    const int cached = g_sms[dev].load(std::memory_order_relaxed);
    if (cached > 0) return cached;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  if (dev < kMaxDevices) g_sms[dev].store(n, std::memory_order_relaxed);
  return n;
}

// ------------------------------------------------------------ merge_state

namespace {
// Launches `kern` as a programmatic dependent of the kernel before it on the
// stream: its CTAs may become resident while that kernel finishes.  Every
// kernel launched this way executes griddepcontrol.wait before it touches
// memory, so the dependence on the previous kernel's results is kept.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// The per-row merge (few rows, many parts): one CTA per row.
template <typename TI, typename TO>
cudaError_t launch_parts(const MergeArgs& a, unsigned rows, cudaStream_t st) {
  // D = 64, 128: the shuffle-reduced kernel; other D (D = 256 measured faster
  // with the shared-memory reduction in the decode's dependent launch)
  if (a.D == 64) return launch_pdl(merge_parts_shfl_kernel<TI, TO, 8>, dim3(rows), dim3(256), 0, st, a);
  if (a.D == 128) return launch_pdl(merge_parts_shfl_kernel<TI, TO, 16>, dim3(rows), dim3(256), 0, st, a);
  return launch_pdl(merge_state_parts_kernel<TI, TO>, dim3(rows), dim3(256), 0, st, a);
}
}  // namespace

namespace {
// Many-row merge with D / 8 = VPR: one thread per SKV_MERGE_SLICES slices,
// 256 threads a block; 32-bit row arithmetic when the slice count fits.
template <typename TI, typename TO, int VPR>
cudaError_t launch_rows(const MergeArgs& a, cudaStream_t st) {
  const dim3 blocks(static_cast<unsigned>((a.n_vec / SKV_MERGE_SLICES + 255) / 256));
  if (a.n_vec < (int64_t(1) << 31) - 256 && static_cast<int64_t>(a.B) * a.H * a.S * a.D < (int64_t(1) << 31))
    return launch_pdl(merge_rows_kernel<TI, TO, VPR, false>, blocks, dim3(256), 0, st, a);
  return launch_pdl(merge_rows_kernel<TI, TO, VPR, true>, blocks, dim3(256), 0, st, a);
}
}  // namespace

int launch_merge_state(const void* o_parts, const float* lse_parts, void* out, float* lse, int P, int B, int H,
                       int S, int D, int layout_bsh, skv_dtype parts_dt, skv_dtype out_dt,
                       int64_t part_stride_o, int64_t part_stride_lse, skv_stream_t stream) {
  MergeArgs a;
  a.o_parts = o_parts;
  a.lse_parts = lse_parts;
  a.out = out;
  a.lse = lse;
  a.P = P;
  a.B = B;
  a.H = H;
  a.S = S;
  a.D = D;
  a.layout_bsh = layout_bsh;
  a.part_stride_o = part_stride_o;
  a.part_stride_lse = part_stride_lse;
  const int64_t rows = static_cast<int64_t>(B) * H * S;
  a.n_vec = rows * (D / 8);
  if (a.n_vec == 0) return 0;
  const int threads = 256;
  const int sms = sm_count();
  const int64_t blocks = (a.n_vec + threads - 1) / threads;
  if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // few rows and many parts: one CTA per row, parallel over the parts
  const bool per_row = P >= 8 && rows <= 4096 && D <= 2048 && sms > 0;
  // many rows, D in {64, 128, 256}: the kernel specialised on the slices per row
  const int vpr = D / 8;
  const bool coop = !per_row && (vpr == 8 || vpr == 16 || vpr == 32);
  cudaError_t le = cudaSuccess;
#define SKV_MERGE(TI, TO)                                                                   \
  do {                                                                                      \
    if (per_row) le = launch_parts<TI, TO>(a, static_cast<unsigned>(rows), st);            \
    else if (coop && vpr == 8) le = launch_rows<TI, TO, 8>(a, st);                          \
    else if (coop && vpr == 16) le = launch_rows<TI, TO, 16>(a, st);                        \
    else if (coop) le = launch_rows<TI, TO, 32>(a, st);                                     \
    else le = launch_pdl(merge_state_kernel<TI, TO>, dim3(static_cast<unsigned>(blocks)),   \
                         dim3(threads), 0, st, a);                                          \
  } while (0)
  if (parts_dt == SKV_FP32 && out_dt == SKV_BF16) SKV_MERGE(float, __nv_bfloat16);
  else if (parts_dt == SKV_FP32 && out_dt == SKV_FP16) SKV_MERGE(float, __half);
  else if (parts_dt == SKV_FP32 && out_dt == SKV_FP32) SKV_MERGE(float, float);
  else if (parts_dt == SKV_BF16 && out_dt == SKV_BF16) SKV_MERGE(__nv_bfloat16, __nv_bfloat16);
  else if (parts_dt == SKV_BF16 && out_dt == SKV_FP32) SKV_MERGE(__nv_bfloat16, float);
  else if (parts_dt == SKV_BF16 && out_dt == SKV_FP16) SKV_MERGE(__nv_bfloat16, __half);
  else if (parts_dt == SKV_FP16 && out_dt == SKV_FP16) SKV_MERGE(__half, __half);
  else if (parts_dt == SKV_FP16 && out_dt == SKV_FP32) SKV_MERGE(__half, float);
  else if (parts_dt == SKV_FP16 && out_dt == SKV_BF16) SKV_MERGE(__half, __nv_bfloat16);
  else return cudaErrorInvalidValue;
#undef SKV_MERGE
  if (le != cudaSuccess) return le;
  return counted(cudaGetLastError(), 1);
}

// ------------------------------------------------------------ decode

namespace {
template <int D, typename T>
int launch_decode_t(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeArgs& a, dim3 grid,
                    cudaStream_t st) {
  using Cfg = DecodeCfg<D>;
  auto kern = decode_split_kernel<D, T>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes);
  if (e != cudaSuccess) return e;
  // programmatic dependent of the previous kernel on the stream (sets up while
  // that kernel finishes; waits before touching memory)
  return counted(launch_pdl(kern, grid, dim3(kDecodeThreads), Cfg::kSmemBytes, st, tk, tv, a), 1);
}
}  // namespace

int launch_decode(const void* q, const void* k, const void* v, void* out, float* lse, float* part_o,
                  float* part_lse, int* counters, const int32_t* kv_len, int B, int Hq, int Hkv, int Lq, int Lkv,
                  int D, float scale, skv_dtype dt, int num_splits, int causal, skv_stream_t stream) {
  const int G = Hq / Hkv;
  DecodeArgs a;
  a.q = q;
  a.out = out;
  a.lse = lse;
  a.part_o = part_o;
  a.part_lse = part_lse;
  a.counters = counters;
  a.kv_len = kv_len;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.Lq = Lq;
  a.Lkv = Lkv;
  a.num_splits = num_splits;
  a.causal = causal;
  a.row_groups = static_cast<int>(ceil_div64(static_cast<int64_t>(G) * Lq, kDecodeRows));
  a.scale_log2 = scale * 1.4426950408889634f;
  // K and V as 2-D [B*Hkv*Lkv rows, D] maps; box = 64 columns x 64 keys
  CUtensorMap tk, tv;
  std::memset(&tk, 0, sizeof(tk));
  std::memset(&tv, 0, sizeof(tv));
  if (Lkv > 0) {  // with no keys the kernel issues no loads and the maps stay unused
    const uint64_t dims[2] = {static_cast<uint64_t>(D), static_cast<uint64_t>(B) * Hkv * Lkv};
    const uint64_t strides[1] = {static_cast<uint64_t>(D) * 2};
    const uint32_t box[2] = {64, kDecodeKeysPerTile};
    int e = make_tmap(&tk, dt, 2, k, dims, strides, box);
    if (e) return e;
    e = make_tmap(&tv, dt, 2, v, dims, strides, box);
    if (e) return e;
  }
  dim3 grid(num_splits, B * Hkv * a.row_groups);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dt == SKV_BF16) {
    if (D == 64) return launch_decode_t<64, __nv_bfloat16>(tk, tv, a, grid, st);
    if (D == 128) return launch_decode_t<128, __nv_bfloat16>(tk, tv, a, grid, st);
    if (D == 256) return launch_decode_t<256, __nv_bfloat16>(tk, tv, a, grid, st);
  } else {
    if (D == 64) return launch_decode_t<64, __half>(tk, tv, a, grid, st);
    if (D == 128) return launch_decode_t<128, __half>(tk, tv, a, grid, st);
    if (D == 256) return launch_decode_t<256, __half>(tk, tv, a, grid, st);
  }
  return cudaErrorInvalidValue;
}

// ------------------------------------------------------------ prefill

namespace {
// 4-D map over q/k/v of one layout: HND dims (D, S, H, B); NHD / TND dims
// (D, H, S, B); box = 64 columns x `rows` rows of one head.
int make_qkv_map(CUtensorMap* m, const void* base, skv_dtype dt, skv_layout layout, int B, int H, int S, int D,
                 uint32_t rows = 128) {
  const uint64_t e = 2;
  uint64_t dims[4], strides[3];
  uint32_t box[4];
  if (layout == SKV_HND) {
    dims[0] = D; dims[1] = S; dims[2] = H; dims[3] = B;
    strides[0] = D * e; strides[1] = static_cast<uint64_t>(S) * D * e; strides[2] = static_cast<uint64_t>(H) * S * D * e;
    box[0] = 64; box[1] = rows; box[2] = 1; box[3] = 1;
  } else {
    dims[0] = D; dims[1] = H; dims[2] = S; dims[3] = B;
    strides[0] = D * e; strides[1] = static_cast<uint64_t>(H) * D * e; strides[2] = static_cast<uint64_t>(S) * H * D * e;
    box[0] = 64; box[1] = 1; box[2] = rows; box[3] = 1;
  }
  return make_tmap(m, dt, 4, base, dims, strides, box);
}

// int8 codes [B, H, S, 128] (HND) as a 4-D map (D, S, H, B), box 128 x 128 rows
int make_i8_map(CUtensorMap* m, const void* base, int B, int H, int S) {
  const uint64_t D = 128;
  const uint64_t dims[4] = {D, static_cast<uint64_t>(S), static_cast<uint64_t>(H), static_cast<uint64_t>(B)};
  const uint64_t strides[3] = {D, static_cast<uint64_t>(S) * D, static_cast<uint64_t>(H) * S * D};
  const uint32_t box[4] = {128, 128, 1, 1};
  return make_tmap_ty(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, base, dims, strides, box);
}

template <int D, typename T, bool kI8 = false>
int launch_prefill_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& to,
                     const PrefillArgs& a, unsigned grid, cudaStream_t st, bool dependent = false) {
  using Cfg = PrefillCfg<D, kI8>;
  auto kern = prefill_kernel<D, T, kI8>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes);
  if (e != cudaSuccess) return e;
  if (!dependent) {
    kern<<<grid, kPfThreads, Cfg::kSmemBytes, st>>>(tq, tk, tv, to, a);
    return counted(cudaGetLastError(), 1);
  }
  // programmatic dependent of the K column-sum kernel: CTAs start while it
  // streams K; only the softmax warps' read of its sums waits for it
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kPfThreads);
  cfg.dynamicSmemBytes = Cfg::kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return counted(cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, to, a), 1);
}

}  // namespace

int launch_prefill(const PrefillLaunch& p, skv_stream_t stream) {
  const bool varlen = p.layout == SKV_TND;
  const int Bm = varlen ? 1 : p.B;       // batch extent of the maps
  CUtensorMap tq, tk, tv;
  int e = make_qkv_map(&tq, p.q, p.dt, p.layout, Bm, p.Hq, p.Sq > 0 ? p.Sq : 1, p.D);
  if (e) return e;
  std::memset(&tk, 0, sizeof(tk));
  std::memset(&tv, 0, sizeof(tv));
  if (p.Sk > 0) {  // with no keys every CTA writes O = 0, LSE = -inf without loads
    e = make_qkv_map(&tk, p.k, p.dt, p.layout, Bm, p.Hkv, p.Sk, p.D);
    if (e) return e;
    e = make_qkv_map(&tv, p.v, p.dt, p.layout, Bm, p.Hkv, p.Sk, p.D);
    if (e) return e;
  }
  // O: the layout of Q, with a multi-chunk call's chunks stacked on the batch axis
  const int nch_o = (varlen || p.nchunks < 1) ? 1 : p.nchunks;
  CUtensorMap to;
  e = make_qkv_map(&to, p.out, p.dt, p.layout, Bm * nch_o, p.Hq, p.Sq > 0 ? p.Sq : 1, p.D);
  if (e) return e;
  PrefillArgs a;
  a.out = p.out;
  a.lse = p.lse;
  a.qscale = nullptr;
  a.kscale = nullptr;
  a.dq = nullptr;
  a.kmean = p.kmean;
  a.kpartial = p.kpartial;
  a.shift_logits = p.shift_logits;
  a.causal = p.causal;
  a.cu_q = p.cu_q;
  a.cu_k = p.cu_k;
  a.order = p.order;
  a.offsets = p.offsets;
  a.B = p.B;
  a.Hq = p.Hq;
  a.Hkv = p.Hkv;
  a.Sq = p.Sq;
  a.Sk = p.Sk;
  a.layout = varlen ? 2 : (p.layout == SKV_HND ? 0 : 1);
  a.scale_log2 = p.scale * 1.4426950408889634f;
  const int nch = (varlen || p.nchunks < 1) ? 1 : p.nchunks;
  if (nch > kMaxKvChunks || (nch > 1 && p.kv_bounds == nullptr)) return cudaErrorInvalidValue;
  a.nchunks = nch;
  a.kvb[0] = 0;
  a.kvb[1] = p.Sk;
  if (nch > 1)
    for (int c = 0; c <= nch; ++c) a.kvb[c] = p.kv_bounds[c];
  int64_t grid;
  if (varlen) {
    // upper bound on sum_b ceil(len_q(b) / 256); surplus CTAs exit at once
    a.nqb = 0;
    grid = static_cast<int64_t>(p.Hq) * (ceil_div64(p.Sq, prefill_rows_per_cta(p.D)) + p.B);
  } else {
    a.nqb = static_cast<int>(ceil_div64(p.Sq, prefill_rows_per_cta(p.D)));
    grid = static_cast<int64_t>(nch) * p.B * p.Hq * a.nqb;
  }
  if (grid <= 0) return 0;
  if (grid > 0x7fffffff) return cudaErrorInvalidValue;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool dep = p.after_kpartial != 0 && p.kpartial != nullptr;
  if (p.dt == SKV_BF16) {
    if (p.D == 64) return launch_prefill_t<64, __nv_bfloat16>(tq, tk, tv, to, a, static_cast<unsigned>(grid), st, dep);
    if (p.D == 128) return launch_prefill_t<128, __nv_bfloat16>(tq, tk, tv, to, a, static_cast<unsigned>(grid), st, dep);
    if (p.D == 256) return launch_prefill_t<256, __nv_bfloat16>(tq, tk, tv, to, a, static_cast<unsigned>(grid), st, dep);
  } else {
    if (p.D == 64) return launch_prefill_t<64, __half>(tq, tk, tv, to, a, static_cast<unsigned>(grid), st, dep);
    if (p.D == 128) return launch_prefill_t<128, __half>(tq, tk, tv, to, a, static_cast<unsigned>(grid), st, dep);
    if (p.D == 256) return launch_prefill_t<256, __half>(tq, tk, tv, to, a, static_cast<unsigned>(grid), st, dep);
  }
  return cudaErrorInvalidValue;
}

namespace {
// K column sums (smooth.cuh): one CTA per unit (256-key chunk, range, kv
// head) on a 1-D grid, as a programmatic dependent of the kernel before it
cudaError_t launch_kmean_partial(const SmoothArgs& a, skv_dtype dt, cudaStream_t st) {
  const int64_t units = static_cast<int64_t>(a.nchunks) * a.Bseq * a.Hkv;
  if (units <= 0) return cudaSuccess;
  if (units > 0x7fffffff) return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>(units));
  if (dt == SKV_BF16) return launch_pdl(kmean_partial_kernel<__nv_bfloat16>, grid, dim3(256), 0, st, a);
  return launch_pdl(kmean_partial_kernel<__half>, grid, dim3(256), 0, st, a);
}
}  // namespace

int launch_prefill_int8(const Int8PrefillLaunch& p, skv_stream_t stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int nqb = static_cast<int>(ceil_div64(p.Sq, kQuantBlock));
  const int nkb = static_cast<int>(ceil_div64(p.Sk, kQuantBlock));
  int launches = 0;
  // fp32 mean of K over the call's keys: per-256-key column sums, then the mean
  SmoothArgs sa;
  sa.k = p.k;
  sa.k_out = nullptr;
  sa.partial = p.kpartial;
  sa.kmean = p.kmean;
  sa.cu_k = nullptr;
  sa.Bseq = p.B;
  sa.Hkv = p.Hkv;
  sa.Sk = p.Sk;
  sa.D = 128;
  sa.nchunks = static_cast<int>(ceil_div64(p.Sk, kSmoothChunk));
  sa.layout = 0;
  sa.kv_ranges = 1;
  sa.kvb[0] = 0;
  sa.kvb[1] = p.Sk;
  {
    const cudaError_t e = launch_kmean_partial(sa, p.dt, st);
    if (e != cudaSuccess) return e;
    kmean_finalize_kernel<<<p.B * p.Hkv, 128, 0, st>>>(sa);
    launches += 2;
  }
  // codes of K - mean and of Q (+ the per-row smoothing shift)
  QuantArgs qa;
  qa.kmean = p.kmean;
  qa.B = p.B;
  qa.Hkv = p.Hkv;
  qa.scale_log2 = p.scale * 1.4426950408889634f;
  qa.x = p.k;
  qa.codes = p.k8;
  qa.scales = p.kscale;
  qa.dq = nullptr;
  qa.H = p.Hkv;
  qa.S = p.Sk;
  qa.nblk = nkb;
  if (p.dt == SKV_BF16) quant_int8_kernel<__nv_bfloat16, false><<<dim3(nkb, p.B * p.Hkv), 256, 0, st>>>(qa);
  else quant_int8_kernel<__half, false><<<dim3(nkb, p.B * p.Hkv), 256, 0, st>>>(qa);
  qa.x = p.q;
  qa.codes = p.q8;
  qa.scales = p.qscale;
  qa.dq = p.dq;
  qa.H = p.Hq;
  qa.S = p.Sq;
  qa.nblk = nqb;
  if (p.dt == SKV_BF16) quant_int8_kernel<__nv_bfloat16, true><<<dim3(nqb, p.B * p.Hq), 256, 0, st>>>(qa);
  else quant_int8_kernel<__half, true><<<dim3(nqb, p.B * p.Hq), 256, 0, st>>>(qa);
  launches += 2;
  cudaError_t le = cudaGetLastError();
  if (le != cudaSuccess) return le;
  count_launches(launches);
  // the prefill over the codes (V stays 16-bit)
  CUtensorMap tq, tk, tv;
  int e = make_i8_map(&tq, p.q8, p.B, p.Hq, p.Sq);
  if (e) return e;
  e = make_i8_map(&tk, p.k8, p.B, p.Hkv, p.Sk);
  if (e) return e;
  e = make_qkv_map(&tv, p.v, p.dt, SKV_HND, p.B, p.Hkv, p.Sk, 128);
  if (e) return e;
  CUtensorMap to;
  e = make_qkv_map(&to, p.out, p.dt, SKV_HND, p.B, p.Hq, p.Sq, 128);
  if (e) return e;
  PrefillArgs a;
  std::memset(&a, 0, sizeof(a));
  a.out = p.out;
  a.lse = p.lse;
  a.qscale = p.qscale;
  a.kscale = p.kscale;
  a.dq = p.dq;
  a.causal = p.causal;
  a.B = p.B;
  a.Hq = p.Hq;
  a.Hkv = p.Hkv;
  a.Sq = p.Sq;
  a.Sk = p.Sk;
  a.layout = 0;
  a.scale_log2 = p.scale * 1.4426950408889634f;
  a.nchunks = 1;
  a.kvb[0] = 0;
  a.kvb[1] = p.Sk;
  a.nqb = static_cast<int>(ceil_div64(p.Sq, kPrefillRowsPerCta));
  const int64_t grid = static_cast<int64_t>(p.B) * p.Hq * a.nqb;
  if (grid <= 0) return 0;
  if (grid > 0x7fffffff) return cudaErrorInvalidValue;
  if (p.dt == SKV_BF16) return launch_prefill_t<128, __nv_bfloat16, true>(tq, tk, tv, to, a, static_cast<unsigned>(grid), st);
  return launch_prefill_t<128, __half, true>(tq, tk, tv, to, a, static_cast<unsigned>(grid), st);
}

int launch_varlen_plan(const int32_t* cu_q, const int32_t* cu_k, int B, int Hq, int rows_per_cta, int32_t* order,
                       int32_t* offsets, skv_stream_t stream) {
  // one block; no more threads than sequences (rounded to a warp): the final
  // scan walks one partial sum per thread
  const int threads = B >= 1024 ? 1024 : ((B + 31) / 32) * 32;
  varlen_plan_kernel<<<1, threads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(cu_q, cu_k, B, Hq, rows_per_cta, order,
                                                                               offsets);
  return counted(cudaGetLastError(), 1);
}

// ------------------------------------------------------------ diagnostics

namespace {
// The prefill's FMA-pipe exp2, elementwise (for tests of its error).
__global__ void exp2_fma_kernel(const float* __restrict__ x, float* __restrict__ y, int64_t n) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (2 * i + 1 < n) {
    float p0, p1;
    poly_exp2_pair(f2_pack(x[2 * i], x[2 * i + 1]), p0, p1);
    y[2 * i] = p0;
    y[2 * i + 1] = p1;
  } else if (2 * i < n) {
    float p0, p1;
    poly_exp2_pair(f2_pack(x[2 * i], 0.f), p0, p1);
    y[2 * i] = p0;
  }
}
}  // namespace

int launch_exp2_fma(const float* x, float* y, int64_t n, skv_stream_t stream) {
  const int64_t pairs = (n + 1) / 2;
  if (pairs == 0) return 0;
  const int64_t blocks = (pairs + 255) / 256;
  if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
  exp2_fma_kernel<<<static_cast<unsigned>(blocks), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(x, y, n);
  return counted(cudaGetLastError(), 1);
}

// ------------------------------------------------------------ smooth_k

int launch_smooth_k(const void* k, void* k_smoothed, float* kmean, float* partial, const int32_t* cu_k, int B,
                    int Hkv, int Sk, int max_len, int D, skv_dtype dt, skv_layout layout, skv_stream_t stream,
                    int kv_ranges, const int32_t* kv_bounds) {
  SmoothArgs a;
  a.k = k;
  a.k_out = k_smoothed;
  a.partial = partial;
  a.kmean = kmean;
  a.cu_k = cu_k;
  a.Hkv = Hkv;
  a.Sk = Sk;
  a.D = D;
  a.layout = layout == SKV_HND ? 0 : (layout == SKV_NHD ? 1 : 2);
  a.kv_ranges = (layout == SKV_TND || kv_ranges < 1) ? 1 : kv_ranges;
  if (a.kv_ranges > kMaxKvChunks || (a.kv_ranges > 1 && kv_bounds == nullptr)) return cudaErrorInvalidValue;
  a.kvb[0] = 0;
  a.kvb[1] = Sk;
  if (a.kv_ranges > 1)
    for (int c = 0; c <= a.kv_ranges; ++c) a.kvb[c] = kv_bounds[c];
  a.Bseq = B * a.kv_ranges;
  a.nchunks = static_cast<int>(ceil_div64(max_len, kSmoothChunk));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (a.nchunks > 0) {
    const cudaError_t e = launch_kmean_partial(a, dt, st);
    if (e != cudaSuccess) return e;
  }
  // the mean itself is needed here only to materialise K'; otherwise the
  // prefill kernel adds up the per-chunk partial sums of its own KV range
  if (k_smoothed != nullptr) kmean_finalize_kernel<<<a.Bseq * Hkv, D, 0, st>>>(a);
  if (k_smoothed != nullptr && a.nchunks > 0) {
    const unsigned units = static_cast<unsigned>(static_cast<int64_t>(a.nchunks) * a.Bseq * Hkv);
    if (dt == SKV_BF16) ksmooth_write_kernel<__nv_bfloat16><<<units, 256, 0, st>>>(a);
    else ksmooth_write_kernel<__half><<<units, 256, 0, st>>>(a);
  }
  const int n = (a.nchunks > 0 ? 1 : 0) + (k_smoothed != nullptr ? 1 : 0) +
                (k_smoothed != nullptr && a.nchunks > 0 ? 1 : 0);
  return counted(cudaGetLastError(), n);
}

}  // namespace skv

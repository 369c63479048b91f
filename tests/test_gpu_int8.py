"""GPU parity of attn_fwd_lse_int8 (INT8 Q K'^T with smooth_k) against the
FP64 oracle's INT8 definition, through the C ABI.

The codes themselves are compared too (read from the documented workspace
sections): Q codes and scales must equal the oracle's bit for bit (the same
fp32 operations on the same 16-bit inputs); K' = K - mean depends on the
mean's fp32 summation order, so a K' code may differ by one where the
oracle's x * 127 / amax lies within a hair of a rounding tie, and nowhere else."""
import numpy as np
import pytest
import torch

import oracle as O
import split_kv_merge_attn_b200 as skv
import workloads as W
from tests._gpu_helpers import check_lse, check_o, nan_empty, vmax

pytestmark = pytest.mark.gpu


def _a256(x):
    return (x + 255) // 256 * 256


def ws_sections(B, Hq, Hkv, Sq, Sk):
    sizes = [((Sk + 255) // 256) * B * Hkv * 128 * 4, B * Hkv * 128 * 4, B * Hq * Sq * 128, B * Hkv * Sk * 128,
             B * Hq * ((Sq + 127) // 128) * 4, B * Hkv * ((Sk + 127) // 128) * 4, B * Hq * Sq * 4]
    offs, o = [], 0
    for sz in sizes:
        offs.append((o, sz))
        o += _a256(sz)
    return offs, o


def run_int8(d, causal=False):
    q, k, v = d["q"].cuda(), d["k"].cuda(), d["v"].cuda()
    B, Hq, Sq, D = q.shape
    _, Hkv, Sk, _ = k.shape
    nbytes = skv.attn_fwd_lse_int8_workspace(B, Hq, Hkv, Sq, Sk, D)
    offs, total = ws_sections(B, Hq, Hkv, Sq, Sk)
    assert nbytes == total
    ws = torch.full((nbytes,), 0x5A, dtype=torch.uint8, device="cuda")
    out = nan_empty(q.shape, q.dtype)
    lse = nan_empty((B, Hq, Sq), torch.float32)
    out, lse = skv.attn_fwd_lse_int8(q, k, v, d["scale"], causal=causal, out=out, lse=lse, workspace=ws)
    torch.cuda.synchronize()
    assert skv.device_error() == 0
    wh = ws.cpu().numpy()

    def sec(i, dtype, shape):
        o, sz = offs[i]
        return wh[o:o + sz].view(dtype).reshape(shape)
    codes = {"q8": sec(2, np.int8, (B, Hq, Sq, 128)), "k8": sec(3, np.int8, (B, Hkv, Sk, 128)),
             "qs": sec(4, np.float32, (B, Hq, -1)), "ks": sec(5, np.float32, (B, Hkv, -1)),
             "mean": sec(1, np.float32, (B, Hkv, 128))}
    return out, lse, codes


def oracle_int8(d, causal=False):
    q, k, v = O.to_f64(d["q"]), O.to_f64(d["k"]), O.to_f64(d["v"])
    B, Hq, Sq, D = q.shape
    Hkv, Sk = k.shape[1], k.shape[2]
    G = Hq // Hkv
    o = np.zeros((B, Hq, Sq, D))
    l = np.zeros((B, Hq, Sq))
    for b in range(B):
        for h in range(Hq):
            if causal:
                counts = O.causal_key_counts(Sq, Sk)
                # the codes and the mean are those of the call's whole key range; each row
                # sees its first counts[i] keys
                mu = np.float32(O.kv_mean(k[b, h // G].astype(np.float32)))
                kp = (k[b, h // G].astype(np.float32) - mu[None]).astype(np.float32)
                qc, qs = O.quantize_int8_blocks(q[b, h])
                kc, ks = O.quantize_int8_blocks(kp)
                qd = qc * np.repeat(qs.astype(np.float64), 128)[:Sq, None]
                kd = kc * np.repeat(ks.astype(np.float64), 128)[:Sk, None]
                ob, lb = O.attention_rows(qd, kd, v[b, h // G], d["scale"], counts)
                lb = lb + O.smooth_shift(q[b, h].astype(np.float32), mu.astype(np.float64), d["scale"])
            else:
                ob, lb = O.int8_attention_rows(q[b, h], k[b, h // G], v[b, h // G], d["scale"])
            o[b, h], l[b, h] = ob, lb
    return o, l


def check_codes(d, codes):
    q = O.to_f64(d["q"]).astype(np.float32)
    k = O.to_f64(d["k"]).astype(np.float32)
    B, Hq, Sq, _ = q.shape
    Hkv = k.shape[1]
    for b in range(B):
        for h in range(Hq):
            qc, qs = O.quantize_int8_blocks(q[b, h])
            assert np.array_equal(codes["q8"][b, h], qc), (b, h)
            assert np.array_equal(codes["qs"][b, h], qs), (b, h)
        for h in range(Hkv):
            mu = np.float32(O.kv_mean(k[b, h]))
            assert np.allclose(codes["mean"][b, h], mu, rtol=1e-5, atol=1e-6)
            kp = (k[b, h] - mu[None]).astype(np.float32)
            kc, ks = O.quantize_int8_blocks(kp)
            np.testing.assert_allclose(codes["ks"][b, h], ks, rtol=3e-7)
            diff = codes["k8"][b, h].astype(int) - kc.astype(int)
            assert np.abs(diff).max() <= 1
            if np.any(diff):
                # only where x * 127 / amax sits at a rounding tie within the mean's rounding
                amax = np.repeat([np.abs(kp[i:i + 128]).max() for i in range(0, kp.shape[0], 128)],
                                 128)[:kp.shape[0], None].astype(np.float32)
                r = kp * (np.float32(127.0) / amax)
                near = np.abs(np.abs(r - np.floor(r)) - 0.5) < 1e-3
                assert np.all(near[diff != 0])


@pytest.mark.parametrize("Sq,Sk,Hq,Hkv", [(256, 1024, 4, 2), (300, 777, 4, 4), (129, 129, 2, 1), (1, 300, 8, 2)])
def test_int8_matches_oracle_int8(Sq, Sk, Hq, Hkv):
    d = W.dense_case(1, Hq, Hkv, Sq, Sk, 128, seed=Sq + Sk, k_offset=0.5, q_mult=2.0)
    out, lse, codes = run_int8(d)
    check_codes(d, codes)
    o_ref, l_ref = oracle_int8(d)
    check_o(out, o_ref, vmax(d["v"]))
    check_lse(lse, l_ref)


def test_int8_close_to_exact_attention():
    """The quantization error itself (reported, loosely bounded): smoothed K
    keeps the LSE within a few hundredths of the exact one."""
    d = W.dense_case(2, 4, 2, 512, 2048, 128, seed=3, k_offset=2.0)
    out, lse, _ = run_int8(d)
    o_ex, l_ex = O.dense(d["q"], d["k"], d["v"], d["scale"])
    assert float(np.abs(lse.double().cpu().numpy() - l_ex).max()) < 0.05
    assert float(np.abs(out.double().cpu().numpy() - o_ex).max()) < 0.05 * vmax(d["v"])


def test_int8_fp16_and_causal():
    d = W.dense_case(1, 4, 2, 384, 640, 128, seed=8, dtype="fp16", k_offset=0.5)
    out, lse, _ = run_int8(d, causal=True)
    o_ref, l_ref = oracle_int8(d, causal=True)
    check_o(out, o_ref, vmax(d["v"]))
    check_lse(lse, l_ref)


def test_int8_full_size_chunk_sampled():
    """One KV chunk of the chunked workload (B=1, H=16, Sq=Sk=4096, D=128,
    K ~ randn + 0.5): every row of one head against the oracle's INT8
    definition."""
    c = W.config5(Sk=4096, n_chunks=1)
    q, k, v = c["q"].cuda(), c["k"].cuda(), c["v"].cuda()
    out, lse = skv.attn_fwd_lse_int8(q, k, v, c["scale"])
    torch.cuda.synchronize()
    assert skv.device_error() == 0
    for h in (0, 11):
        ob, lb = O.int8_attention_rows(O.to_f64(c["q"][0, h]), O.to_f64(c["k"][0, h]), O.to_f64(c["v"][0, h]),
                                       c["scale"])
        check_o(out[0, h], ob, vmax(c["v"]))
        check_lse(lse[0, h], lb)

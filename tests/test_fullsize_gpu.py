"""Parity at the benchmark workloads' full sizes, in the launch configuration
the benchmark uses (automatic split counts, whole chunks), on sampled outputs
the oracle computes one by one:

* Llama-2-7B-shaped MHA decode at 32K context (needle keys planted in the
  retrieval heads), every query head of one layer;
* Llama-3-8B-shaped GQA decode at 128K context, batch 1 and batch 4, and 128
  fused decode steps (append + attend) with the streaming rings checked after;
* the 32K-token GQA pre-fill in 4K chunks (sampled rows of every chunk and head);
* the 1M-token INT4 GQA decode (one retrieval and one streaming KV head).

Streaming heads are checked against the oracle given only the sink and recent
positions, retrieval heads against the full history.
"""

import os

import numpy as np
import pytest
import torch

from oracle import attention as OA
from oracle import cache as OC
from oracle import int4 as OQ
from head_split_kv_decode_b200 import synth
from head_split_kv_decode_b200.cache import DuoCache

from _util import assert_parity, f64

pytestmark = pytest.mark.gpu

torch.set_num_threads(max(1, os.cpu_count() or 1))


def _fill_decode(w, B, layer=0, chunk=16384):
    """One-layer cache of workload w filled to its context, one decode token
    appended; returns (cache, q, out, mask_row)."""
    mask = synth.workload_mask(w)
    row = mask[layer]
    dt = synth.io_dtype(w)
    cache = DuoCache(1, B, w.n_q_heads, w.n_kv_heads, w.head_dim, w.kv_dtype, w.context + 1,
                     row[None], w.S, w.R)
    for p0 in range(0, w.context + 1, chunk):
        pos = range(p0, min(w.context + 1, p0 + chunk))
        k = synth.history(w, layer, "k", range(B), pos, device="cuda", mask_row=row).to(dt)
        v = synth.history(w, layer, "v", range(B), pos, device="cuda", mask_row=row).to(dt)
        cache.append(0, k.contiguous(), v.contiguous())
    assert cache.seq_len(0) == w.context + 1
    q = synth.queries(w, layer, range(B), [w.context], device="cuda")[:, 0].to(dt).contiguous()
    out = cache.decode(0, q)
    torch.cuda.synchronize()
    return cache, q, out, row


def _oracle_head(w, layer, b, h, row, q, quantised=False, t=None):
    """fp64 oracle for the G query heads of KV head h, batch row b, at position
    t (default: the context length)."""
    t = w.context if t is None else t
    retrieval = bool(row[h])
    if retrieval:
        keys = np.arange(t + 1)
    else:
        keys = np.unique(np.concatenate([np.arange(min(w.S, t + 1)),
                                         np.arange(max(0, t + 1 - w.R), t + 1)]))
    dt = synth.io_dtype(w)
    out = []
    kv = []
    for which in ("k", "v"):
        x = synth.history(w, layer, which, [b], keys, heads=[h], mask_row=row).to(dt)[0, :, 0]
        if quantised:
            codes, sc, zp = OQ.quantize_int4(x.float().numpy())
            kv.append(OQ.dequantize_int4(codes, sc, zp))
        else:
            kv.append(x.double().numpy())
    G = w.group
    qr = q[b, h * G:(h + 1) * G].detach().cpu().double().numpy()
    return OA.attend_head(qr, np.full(G, t), kv[0], kv[1], keys, retrieval, w.S, w.R,
                          OA.default_scale(w.head_dim))


def test_llama2_mha_32k_decode_all_heads():
    w = synth.WORKLOADS["llama2_7b_mha_32k"]
    cache, q, out, row = _fill_decode(w, 1)
    assert cache.decode_splits(0) > 1
    got = out[0].float().cpu()
    ref = np.stack([_oracle_head(w, 0, 0, h, row, q)[0] for h in range(w.n_kv_heads)])
    assert_parity(got, ref, "bf16", "32K MHA decode")


@pytest.mark.parametrize("B,rows", [(1, [0]), (4, [0, 3])])
def test_llama3_gqa_128k_decode(B, rows):
    w = synth.WORKLOADS["llama3_8b_gqa_128k"]
    cache, q, out, row = _fill_decode(w, B)
    for b in rows:
        got = out[b].float().cpu()
        ref = np.concatenate([_oracle_head(w, 0, b, h, row, q) for h in range(w.n_kv_heads)])
        assert_parity(got, ref, "bf16", "128K GQA decode B=%d b=%d" % (B, b))


def test_llama3_gqa_128k_128_fused_decode_steps():
    """128 decode steps with ring-buffer append/evict at 128K, batch 1: each
    step appends its token and attends in one fused launch.  Sampled steps
    match the oracle (one retrieval and one streaming KV head), and after the
    last step a streaming head's slot buffers hold the sinks and the last R
    tokens bit for bit (the ring has advanced 128 slots)."""
    w = synth.WORKLOADS["llama3_8b_gqa_128k"]
    steps, n0, G = 128, w.context, w.group
    row = synth.workload_mask(w)[0]
    dt = synth.io_dtype(w)
    cache = DuoCache(1, 1, w.n_q_heads, w.n_kv_heads, w.head_dim, w.kv_dtype, n0 + steps,
                     row[None], w.S, w.R)
    for p0 in range(0, n0, 16384):
        pos = range(p0, min(n0, p0 + 16384))
        k = synth.history(w, 0, "k", [0], pos, device="cuda", mask_row=row).to(dt)
        v = synth.history(w, 0, "v", [0], pos, device="cuda", mask_row=row).to(dt)
        cache.append(0, k.contiguous(), v.contiguous())
    ret = [h for h in range(w.n_kv_heads) if row[h]][0]
    strm = [h for h in range(w.n_kv_heads) if not row[h]][0]
    for s_ in range(steps):
        t = n0 + s_
        k = synth.history(w, 0, "k", [0], [t], device="cuda", mask_row=row)[:, 0].to(dt).contiguous()
        v = synth.history(w, 0, "v", [0], [t], device="cuda", mask_row=row)[:, 0].to(dt).contiguous()
        q = synth.queries(w, 0, [0], [t], device="cuda")[:, 0].to(dt).contiguous()
        out = cache.step(0, q, k, v)
        if s_ in (0, 1, 77, steps - 1):
            got = out[0].float().cpu()
            for h in (ret, strm):
                ref = _oracle_head(w, 0, 0, h, row, q, t=t)
                assert_parity(got[h * G:(h + 1) * G], ref, "bf16", "step %d head %d" % (s_, h))
    assert cache.seq_len(0) == n0 + steps
    torch.cuda.synchronize()
    idx = cache.layout(0).packed_index[strm]
    for which, name in (("k", "str_k"), ("v", "str_v")):
        hist = synth.history(w, 0, which, [0], range(n0 + steps), heads=[strm], mask_row=row)
        hist = hist.to(dt)[0, :, 0].contiguous().view(torch.uint8).numpy()
        exp, filled = OC.expected_streaming_buffer(hist, w.S, w.R)
        got = cache.region(0, name)[0, idx].cpu().numpy()
        assert filled.all()
        np.testing.assert_array_equal(got[:w.S + w.R], exp)


def test_llama3_gqa_prefill_32k_sampled_rows():
    w = synth.WORKLOADS["llama3_8b_gqa_prefill_32k"]
    mask = synth.workload_mask(w)[:1]
    C, n = w.chunk, w.context
    cache = DuoCache(1, 1, w.n_q_heads, w.n_kv_heads, 128, "bf16", n, mask, w.S, w.R)
    K = synth.history(w, 0, "k", [0], range(n), device="cuda").to(torch.bfloat16)
    V = synth.history(w, 0, "v", [0], range(n), device="cuda").to(torch.bfloat16)
    Q = synth.queries(w, 0, [0], range(n), device="cuda").to(torch.bfloat16)
    outs = []
    for c0 in range(0, n, C):
        sl = slice(c0, c0 + C)
        outs.append(cache.prefill(0, Q[:, sl].contiguous(), K[:, sl].contiguous(),
                                  V[:, sl].contiguous()).cpu())
        cache.append(0, K[:, sl].contiguous(), V[:, sl].contiguous())
    torch.cuda.synchronize()
    Kd, Vd, Qd = f64(K), f64(V), f64(Q)
    g = torch.Generator().manual_seed(4)
    base_rows = [0, 1, 63, 64, 127, 128, 255, 256, w.R - 1, w.R, C - 2, C - 1]
    for ci, c0 in enumerate(range(0, n, C)):
        rows = np.unique(base_rows + torch.randint(0, C, (6,), generator=g).tolist())
        ref = OA.prefill_reference(Qd[:, c0:c0 + C], Kd, Vd, c0, mask[0].numpy(), w.S, w.R,
                                   rows=rows)
        assert_parity(outs[ci][:, rows], ref, "bf16", "prefill chunk %d" % ci)


def test_llama3_int4_1m_decode_sampled_heads():
    w = synth.WORKLOADS["llama3_8b_gqa_int4_1m"]
    cache, q, out_bf16, row = _fill_decode(w, 1, chunk=65536)
    cache.set_decode_output(torch.float32)
    out = cache.decode(0, q)
    torch.cuda.synchronize()
    ret = [h for h in range(w.n_kv_heads) if row[h]][:1]
    strm = [h for h in range(w.n_kv_heads) if not row[h]][:1]
    G = w.group
    worst = 0.0
    for h in ret + strm:
        got = out[0, h * G:(h + 1) * G].cpu()
        ref = _oracle_head(w, 0, 0, h, row, q, quantised=True)
        mx, _ = assert_parity(got, ref, "int4", "1M INT4 decode head %d (fp32 output)" % h)
        worst = max(worst, mx)
        assert_parity(out_bf16[0, h * G:(h + 1) * G].cpu(), ref, "int4_bf16",
                      "1M INT4 decode head %d (bf16 output)" % h)
    print("1M INT4 decode: max |err| %.3g (fp32 output)" % worst)

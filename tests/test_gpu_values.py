"""GPU parity of the value path at the edges of its arithmetic (through the
C ABI, against the CPU oracle at |gpu - oracle| <= 2e-3 + 1e-2 |oracle|):

  * value magnitudes from 1e-3 to 1e4 (the kernel carries value weights in
    16-bit fixed point, scaled to the largest value scale seen and to each
    group's own largest weight), for 4-bit and 2-bit cells, flat and peaky
    queries, tau in {0, 1e-3, 1e-2}.  Attention is linear in V, so values
    scaled by c give outputs scaled by c; the tolerance is the same one
    applied to the values divided by c: |gpu - oracle| <= c * 2e-3 +
    1e-2 |oracle| (a fixed 2e-3 would demand ever more relative precision
    as c grows, and none at all as c shrinks);
  * value scales that grow along the sequence by four orders of magnitude
    (the fixed-point scale is lowered mid-stream);
  * one split of 1250 groups with flat attention (every group's integer
    sums land in the fp32 accumulators);
  * the exact current token of a reuse cell's own loop (k_cur, v_cur);
  * two host threads decoding the same kernel build with different shared
    memory sizes at once;
  * the empty selection of the kinds that cannot select (2-bit, bf16, 4-bit
    at tau = inf): zero words and counts written over buffers of ones;
  * a dense selection (tau = 1e-6 on flat attention: nearly every token
    gathers its low plane in pass 2).
"""

import math
import threading

import pytest
import torch

from loopkv_testlib import ATOL, check_cell, mask_buffers, seeded_bf16, store_tensors

pytestmark = pytest.mark.gpu


def _kv(B, n, hkv, d, seed, vscale=1.0, kscale=1.0):
    k = seeded_bf16((B, n, hkv, d), seed, kscale)
    k[:, :, :, 3] = (k[:, :, :, 3].float() * 10).to(torch.bfloat16)    # an outlier key channel
    v = seeded_bf16((B, n, hkv, d), seed + 1, vscale)
    return k, v


def _q(B, H, d, seed, temperature):
    return seeded_bf16((B, H, d), seed, 0.125 * temperature)


def _decode(kv, q, table, lens, tau, k_cur=None, v_cur=None, max_seq_len=0):
    from mixed_precision_kv_loopkv_b200 import loopkv_decode_attention
    sm, sc = mask_buffers(kv, q.shape[0])
    out = loopkv_decode_attention(kv, 0, 0, q, table, lens, tau, 1.0, sel_mask=sm, sel_count=sc,
                                  k_cur=k_cur, v_cur=v_cur, max_seq_len=max_seq_len)
    torch.cuda.synchronize()
    return out, sm, sc


@pytest.mark.parametrize("kind", ["q4", "q2"])
@pytest.mark.parametrize("vscale", [1e-3, 1.0, 250.0, 1e4])
@pytest.mark.parametrize("temperature", [1.0, 8.0])
def test_value_scale_extremes(kind, vscale, temperature):
    lens = [100, 2000, 4097]
    k, v = _kv(3, 4097, 2, 128, seed=40, vscale=vscale)
    kv, table, lens_d = store_tensors(kind, k, v, lens)
    q = _q(3, 2, 128, 41, temperature)
    pairs = [(b, h) for b in range(3) for h in range(2)]
    for tau in (0.0, 1e-3, 1e-2):
        out, sm, sc = _decode(kv, q, table, lens_d, tau)
        assert torch.isfinite(out.float()).all()
        check_cell(kv, [kind], 0, {0: (k, v)}, q, table, lens_d, tau, 1.0, pairs, out=out, sel_mask=sm,
                   sel_count=sc, atol=ATOL * vscale)


@pytest.mark.parametrize("kind", ["q4", "q2"])
@pytest.mark.parametrize("d", [64, 128])
def test_value_scale_growing_along_the_sequence(kind, d):
    """Value magnitudes rise 1e-2 -> 1e2 along the context: every warp meets
    larger scales than the ones it started with (tolerance for values of
    scale 100, as above)."""
    n = 3000
    k, v = _kv(2, n, 2, d, seed=42)
    ramp = torch.logspace(-2, 2, n, device="cuda").view(1, n, 1, 1)
    v = (v.float() * ramp).to(torch.bfloat16)
    kv, table, lens_d = store_tensors(kind, k, v, [n, 1777])
    q = _q(2, 2, d, 43, 1.0)
    for tau in (0.0, 0.01, math.inf):
        out, sm, sc = _decode(kv, q, table, lens_d, tau)
        check_cell(kv, [kind], 0, {0: (k, v)}, q, table, lens_d, tau, 1.0, [(0, 0), (0, 1), (1, 0), (1, 1)],
                   out=out, sel_mask=sm, sel_count=sc, atol=ATOL * 100.0)


def test_long_split():
    """One split of 40000 tokens (1250 groups, over 300 per warp) with flat
    attention: every group contributes, and the result still matches."""
    n = 40000
    k, v = _kv(1, n, 1, 128, seed=44)
    kv, table, lens_d = store_tensors("q2", k, v, [n], splits=1)
    q = _q(1, 1, 128, 45, 0.5)                 # flat attention: every weight counts
    out, sm, sc = _decode(kv, q, table, lens_d, 0.01)
    check_cell(kv, ["q2"], 0, {0: (k, v)}, q, table, lens_d, 0.01, 1.0, [(0, 0)], out=out, sel_mask=sm,
               sel_count=sc)


@pytest.mark.parametrize("kind", ["q4", "q2", "bf16"])
@pytest.mark.parametrize("d", [64, 128])
def test_current_token(kind, d):
    """k_cur, v_cur: one exact token after the stored ones; ragged lengths
    including an empty sequence (the output is then v_cur) and a single
    stored token, the low-plane selection taken in the n + 1 softmax."""
    lens = [0, 1, 31, 33, 700, 2049]
    B, hkv = len(lens), 2
    k, v = _kv(B, max(lens), hkv, d, seed=46)
    kc = seeded_bf16((B, hkv, d), 47, 1.0)
    vc = seeded_bf16((B, hkv, d), 48, 1.0)
    kv, table, lens_d = store_tensors(kind, k, v, lens)
    pairs = [(b, h) for b in range(B) for h in range(hkv)]
    for temperature in (1.0, 6.0):
        q = _q(B, hkv, d, 49, temperature)
        for tau in (0.0, 0.01, math.inf):
            out, sm, sc = _decode(kv, q, table, lens_d, tau, k_cur=kc, v_cur=vc)
            check_cell(kv, [kind], 0, {0: (k, v)}, q, table, lens_d, tau, 1.0, pairs, out=out, sel_mask=sm,
                       sel_count=sc, current=(kc, vc))
    assert torch.allclose(out[0].float(), vc[0].float(), rtol=0, atol=0)


@pytest.mark.parametrize("g", [2, 4])
def test_current_token_grouped(g):
    lens = [5, 300, 1500]
    B, hkv, d = len(lens), 2, 128
    k, v = _kv(B, max(lens), hkv, d, seed=50)
    kc, vc = seeded_bf16((B, hkv, d), 51), seeded_bf16((B, hkv, d), 52)
    kv, table, lens_d = store_tensors("q4", k, v, lens, heads=g * hkv)
    q = _q(B, g * hkv, d, 53, 4.0)
    out, sm, sc = _decode(kv, q, table, lens_d, 0.01, k_cur=kc, v_cur=vc)
    check_cell(kv, ["q4"], 0, {0: (k, v)}, q, table, lens_d, 0.01, 1.0,
               [(b, h) for b in range(B) for h in range(g * hkv)], out=out, sel_mask=sm, sel_count=sc,
               current=(kc, vc))


def test_two_threads_different_lengths():
    """Two host threads decode the same cell with different max_seq_len (so
    different dynamic shared memory on the same kernel build) on their own
    streams, many times each; every result equals the serial one."""
    from mixed_precision_kv_loopkv_b200 import loopkv_decode_attention
    lens_long, lens_short = [4096, 100, 2000, 33], [256, 96, 256, 32]
    k, v = _kv(4, 4096, 2, 128, seed=54)
    kv, table, lens_l = store_tensors("q4", k, v, lens_long)
    lens_s = torch.tensor(lens_short, dtype=torch.int32, device="cuda")
    q = _q(4, 2, 128, 55, 2.0)
    ref_l = loopkv_decode_attention(kv, 0, 0, q, table, lens_l, 0.01, max_seq_len=4096)
    ref_s = loopkv_decode_attention(kv, 0, 0, q, table, lens_s, 0.01, max_seq_len=256)
    torch.cuda.synchronize()
    errors, bad = [], []

    def worker(lens, max_len, ref):
        try:
            stream = torch.cuda.Stream()
            out = torch.empty_like(q)
            with torch.cuda.stream(stream):
                for _ in range(200):
                    loopkv_decode_attention(kv, 0, 0, q, table, lens, 0.01, out=out, max_seq_len=max_len,
                                            stream=stream)
                    if not torch.equal(out, ref):
                        bad.append(max_len)
            stream.synchronize()
        except Exception as e:  # a failed launch raises LoopKVError
            errors.append(repr(e))

    threads = [threading.Thread(target=worker, args=a) for a in
               ((lens_l, 4096, ref_l), (lens_s, 256, ref_s))]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors
    assert not bad


@pytest.mark.parametrize("kind,tau", [("q2", 0.01), ("bf16", 0.01), ("q4", math.inf)])
@pytest.mark.parametrize("with_mask", [True, False])
def test_empty_selection_is_written(kind, tau, with_mask):
    """Kinds that cannot select (2-bit, bf16) and a 4-bit cell at tau = inf
    write zero selection words for every group of each sequence and a zero
    count, over buffers that start out filled with ones (and a count alone,
    without words, is still written)."""
    from mixed_precision_kv_loopkv_b200 import loopkv_decode_attention
    lens = [1, 31, 700, 3000]
    k, v = _kv(len(lens), max(lens), 2, 128, seed=56)
    kv, table, lens_d = store_tensors(kind, k, v, lens)
    q = _q(len(lens), 2, 128, 57, 8.0)
    sm, sc = mask_buffers(kv, len(lens))
    sm.fill_(-1)
    sc.fill_(-1)
    out = loopkv_decode_attention(kv, 0, 0, q, table, lens_d, tau, 1.0, sel_mask=sm if with_mask else None,
                                  sel_count=sc)
    torch.cuda.synchronize()
    assert torch.all(sc == 0)
    if with_mask:
        for b, n in enumerate(lens):
            assert torch.all(sm[b, :, : (n + 31) // 32] == 0)
            assert torch.all(sm[b, :, (n + 31) // 32:] == -1)   # words past the sequence are not touched
    check_cell(kv, [kind], 0, {0: (k, v)}, q, table, lens_d, tau, 1.0,
               [(b, h) for b in range(len(lens)) for h in range(2)], out=out)


@pytest.mark.parametrize("d", [64, 128])
def test_dense_selection(d):
    """tau = 1e-6 on flat attention selects nearly every token: the gather of
    pass 2 then walks every group of every warp, four rows per round trip;
    the output matches the oracle and, within the tolerance, the uniform
    4-bit result (tau = 0)."""
    lens = [1, 33, 700, 2000]
    k, v = _kv(len(lens), max(lens), 2, d, seed=58)
    kv, table, lens_d = store_tensors("q4", k, v, lens)
    q = _q(len(lens), 2, d, 59, 0.5)
    pairs = [(b, h) for b in range(len(lens)) for h in range(2)]
    out, sm, sc = _decode(kv, q, table, lens_d, 1e-6)
    check_cell(kv, ["q4"], 0, {0: (k, v)}, q, table, lens_d, 1e-6, 1.0, pairs, out=out, sel_mask=sm,
               sel_count=sc)
    assert int(sc.sum()) > 0.99 * 2 * sum(lens)
    full, _, _ = _decode(kv, q, table, lens_d, 0.0)
    assert torch.allclose(out.float(), full.float(), rtol=1e-2, atol=ATOL)

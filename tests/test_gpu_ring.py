"""GPU parity of the sequence-sharded (ring) causal forward, through the C
ABI, against the float64 oracle's causal attention over the whole sequence.

The W ranks of a ring are emulated one after another in this process: each
rank's steps receive the K/V chunks that the ring would deliver at that step
(rank (r - s) mod W's), so the kernels, the log-sum-exp merges and the
zigzag schedule run exactly as on W GPUs; only the transport (tested over
gloo in test_ring_cpu.py) is left out.  The driver itself runs on one rank
(no torch.distributed).  Chunks of 300 tokens leave ragged 128-row tiles."""
import numpy as np
import pytest
import torch

import oracle
from causal_attention_swa_b200 import inputs, ring, swa
from _compare import check_bf16, check_f32, check_lse, to_f64

pytestmark = pytest.mark.gpu


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _emulate(q, k, v, world):
    chunks = {r: [ring.zigzag_split(t, r, world) for t in (q, k, v)] for r in range(world)}
    outs, lses = [], []
    for r in range(world):
        (qa, qb), _, _ = chunks[r]
        state = ring.RingForwardState((qa, qb), r, world)
        for s in range(world):
            _, (ka, kb), (va, vb) = chunks[(r - s) % world]
            state.step(s, torch.stack((ka, kb, va, vb)))
        (oa, ob), (la, lb) = state.result()
        outs.append((oa, ob))
        lses.append((la.unsqueeze(-1), lb.unsqueeze(-1)))
    torch.cuda.synchronize()
    assert swa.get_device_error() == swa.SWA_OK
    return ring.zigzag_join(outs, world), ring.zigzag_join(lses, world).squeeze(-1)


def _bf16_case(world, chunk, seed, inf_at=()):
    N = 2 * world * chunk
    qb, kb, vb = inputs.attn_bf16_batch(1, 2, N, seed=seed)
    vb = vb.copy()
    for (h, t, d) in inf_at:
        vb[0, h, t, d] = 0x7F80  # +inf
    return (qb, kb, vb), N


@pytest.mark.parametrize("world", [2, 3])
def test_ring_bf16_emulated_ranks_match_the_oracle(world):
    (qb, kb, vb), N = _bf16_case(world, 300, seed=40 + world)
    out, lse = _emulate(_dev(qb), _dev(kb), _dev(vb), world)
    w_out, w_lse = oracle.attn_fwd(*(inputs.bf16_to_f64(b) for b in (qb, kb, vb)))
    check_bf16(out, w_out, f"ring out (W={world})")
    check_lse(lse, w_lse, f"ring lse (W={world})")


def test_ring_bf16_infinity_in_v_keeps_the_absent_row_classes():
    # +inf in a key of chunk 0 (every later row sees it) and of chunk 2
    (qb, kb, vb), N = _bf16_case(2, 300, seed=47, inf_at=[(0, 10, 5), (1, 650, 7)])
    out, lse = _emulate(_dev(qb), _dev(kb), _dev(vb), 2)
    w_out, w_lse = oracle.attn_fwd(*(inputs.bf16_to_f64(b) for b in (qb, kb, vb)))
    check_bf16(out, w_out, "ring out with +inf")
    o = to_f64(out)
    assert np.isposinf(o[0, 0, 10:, 5]).all() and np.isfinite(o[0, 0, :10, 5]).all()
    assert np.isposinf(o[0, 1, 650:, 7]).all() and np.isfinite(o[0, 1, :650, 7]).all()


def test_ring_driver_on_one_rank_matches_the_oracle():
    (qb, kb, vb), N = _bf16_case(1, 700, seed=44)
    q, k, v = _dev(qb), _dev(kb), _dev(vb)
    (qa, qb2), (ka, kb2), (va, vb2) = (ring.zigzag_split(t, 0, 1) for t in (q, k, v))
    (oa, ob), (la, lb) = ring.ring_attn_fwd(qa, qb2, ka, kb2, va, vb2)
    torch.cuda.synchronize()
    out = ring.zigzag_join([(oa, ob)], 1)
    lse = ring.zigzag_join([(la.unsqueeze(-1), lb.unsqueeze(-1))], 1).squeeze(-1)
    w_out, w_lse = oracle.attn_fwd(*(inputs.bf16_to_f64(b) for b in (qb, kb, vb)))
    check_bf16(out, w_out, "ring driver out")
    check_lse(lse, w_lse, "ring driver lse")
    # and it equals the single-call forward within the same bound
    ref, ref_lse = swa.attn_fwd(q, k, v, causal=True)
    check_bf16(out, to_f64(ref), "ring driver vs one call", rel=4e-2)


def test_ring_float32_emulated_ranks_match_the_oracle():
    rng = np.random.default_rng(46)
    N = 2 * 2 * 96
    q, k, v = (rng.standard_normal((1, 2, N, 64)) for _ in range(3))
    tq, tk, tv = (torch.from_numpy(a.astype(np.float32)).cuda() for a in (q, k, v))
    out, lse = _emulate(tq, tk, tv, 2)
    w_out, w_lse = oracle.attn_fwd(*(a.astype(np.float32).astype(np.float64) for a in (q, k, v)))
    check_f32(out, w_out, "ring out f32")
    check_f32(lse, w_lse, "ring lse f32")


def test_merge_of_two_key_halves_is_the_whole_row():
    """swa_attn_merge alone: the forward over keys [0, N) equals the merge of
    the forwards over the halves (non-causal), against the oracle."""
    N = 512
    qb, kb, vb = inputs.attn_bf16_batch(1, 3, N, seed=45)
    q, k, v = _dev(qb), _dev(kb), _dev(vb)
    acc = torch.empty((1, 3, N // 2, 64), dtype=torch.float32, device="cuda")
    lacc = torch.empty((1, 3, N // 2), dtype=torch.float32, device="cuda")
    fin = torch.empty((1, 3, N // 2, 64), dtype=torch.bfloat16, device="cuda")
    qh = q[:, :, : N // 2].contiguous()
    for i, sl in enumerate((slice(0, N // 2), slice(N // 2, N))):
        o, l = swa.attn_fwd(qh, k[:, :, sl].contiguous(), v[:, :, sl].contiguous(), causal=False)
        swa.attn_merge(o, l, acc, lacc, first=(i == 0), out_final=fin if i == 1 else None)
    torch.cuda.synchronize()
    # the oracle takes N queries: the first half twice (a non-causal row
    # depends on its own query and all keys only)
    qh64 = inputs.bf16_to_f64(qb)[:, :, : N // 2]
    w_out, w_lse = oracle.attn_fwd(np.concatenate([qh64, qh64], axis=2), inputs.bf16_to_f64(kb),
                                   inputs.bf16_to_f64(vb), causal=False)
    check_bf16(fin, w_out[:, :, : N // 2], "merged out")
    check_bf16(acc, w_out[:, :, : N // 2], "merged accumulator")
    check_lse(lacc, w_lse[:, :, : N // 2], "merged lse")


def _emulate_bwd(q, k, v, out, lse, dout, world):
    """The ring backward's ranks one after another: rank r at step s works on
    the K/V chunks (and the travelling dk, dv sums) of rank (r - s) mod W."""
    def split(t):
        return [ring.zigzag_split(t, r, world) for r in range(world)]
    qs, ks, vs, os_, ds = split(q), split(k), split(v), split(out), split(dout)
    ls = split(lse.unsqueeze(-1))
    sums = {r: torch.zeros((4,) + ks[r][0].shape, dtype=torch.float32, device="cuda")
            for r in range(world)}
    dqs = []
    for r in range(world):
        state = ring.RingBackwardState(qs[r], os_[r], ds[r],
                                       (ls[r][0].squeeze(-1).contiguous(),
                                        ls[r][1].squeeze(-1).contiguous()), r, world)
        for s in range(world):
            src = (r - s) % world
            state.step(s, torch.stack((ks[src][0], ks[src][1], vs[src][0], vs[src][1])),
                       sums[src])
        dqs.append(state.dq())
    dks = [(swa.f32_to_bf16(sums[r][0]), swa.f32_to_bf16(sums[r][1])) for r in range(world)]
    dvs = [(swa.f32_to_bf16(sums[r][2]), swa.f32_to_bf16(sums[r][3])) for r in range(world)]
    torch.cuda.synchronize()
    assert swa.get_device_error() == swa.SWA_OK
    return tuple(ring.zigzag_join(p, world) for p in (dqs, dks, dvs))


@pytest.mark.parametrize("world", [2, 3])
def test_ring_backward_emulated_ranks_match_the_oracle(world):
    """dq, dk, dv of loss = 1/2 sum out^2 over the sharded sequence, with the
    ring forward's stored output as dout, against the oracle's backward at
    that same output (the comparison of the swa_attn_bwd unit test)."""
    (qb, kb, vb), N = _bf16_case(world, 300, seed=50 + world)
    q, k, v = _dev(qb), _dev(kb), _dev(vb)
    out, lse = _emulate(q, k, v, world)
    dq, dk, dv = _emulate_bwd(q, k, v, out, lse, out, world)
    o64 = to_f64(out)
    w_dq, w_dk, w_dv = oracle.attn_bwd(*(inputs.bf16_to_f64(b) for b in (qb, kb, vb)), o64,
                                       out=o64)
    check_bf16(dq, w_dq, f"ring dq (W={world})")
    check_bf16(dk, w_dk, f"ring dk (W={world})")
    check_bf16(dv, w_dv, f"ring dv (W={world})")


def test_ring_backward_driver_on_one_rank_matches_swa_attn_bwd():
    (qb, kb, vb), N = _bf16_case(1, 640, seed=55)
    q, k, v = _dev(qb), _dev(kb), _dev(vb)
    out, lse = swa.attn_fwd(q, k, v, causal=True)
    parts = [ring.zigzag_split(t, 0, 1) for t in (q, k, v, out)]
    la, lb = ring.zigzag_split(lse.unsqueeze(-1), 0, 1)
    lses = (la.squeeze(-1).contiguous(), lb.squeeze(-1).contiguous())
    (dqa, dqb), (dka, dkb), (dva, dvb) = ring.ring_attn_bwd(
        *parts[0], *parts[1], *parts[2], parts[3], parts[3], lses)
    torch.cuda.synchronize()
    got = [ring.zigzag_join([p], 1) for p in ((dqa, dqb), (dka, dkb), (dva, dvb))]
    want = swa.attn_bwd(q, k, v, out, out, lse, causal=True)
    for g, w, name in zip(got, want, ("dq", "dk", "dv")):
        check_bf16(g, to_f64(w), f"ring driver {name} vs one call", rel=4e-2)
    o64 = to_f64(out)
    w_dq, w_dk, w_dv = oracle.attn_bwd(*(inputs.bf16_to_f64(b) for b in (qb, kb, vb)), o64,
                                       out=o64)
    for g, w, name in zip(got, (w_dq, w_dk, w_dv), ("dq", "dk", "dv")):
        check_bf16(g, w, f"ring driver {name}")


def test_backward_accumulate_mode_adds_to_the_sums():
    """swa_attn_bwd_acc twice into the same float32 sums equals twice the
    bf16 backward (within its rounding), and starts from what is there."""
    N = 384
    qb, kb, vb = inputs.attn_bf16_batch(1, 2, N, seed=56)
    q, k, v = _dev(qb), _dev(kb), _dev(vb)
    out, lse = swa.attn_fwd(q, k, v, causal=True)
    ref = [to_f64(t) for t in swa.attn_bwd(q, k, v, out, out, lse, causal=True)]
    sums = [torch.full(q.shape, 0.5, dtype=torch.float32, device="cuda") for _ in range(3)]
    for _ in range(2):
        swa.attn_bwd_acc(q, k, v, out, out, lse, *sums, causal=True)
    torch.cuda.synchronize()
    for s_, r, name in zip(sums, ref, ("dq", "dk", "dv")):
        check_bf16((s_.double().cpu().numpy() - 0.5) / 2.0, r, f"accumulated {name}")

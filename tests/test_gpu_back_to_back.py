"""Micro-steps launched back to back, with no host synchronisation between them.

Consecutive attention launches overlap on the GPU: a launch's CTAs may start while earlier
micro-steps finish, and calls on the same layer buffer are ordered only by per-layer counters
in the workspace (a call reads buffer rows once the earlier calls that wrote them have
scattered, and scatters once the earlier calls that read the rows it overwrites have finished
reading: with one buffer half every earlier call, with two the calls up to the previous
step's call for the same patch).  The other parity tests synchronise
after every call to check the buffer; here every call of a few diffusion steps -- the patch
calls of every layer, text-token queries on every layer after patch 1 and again at the end of
each step -- is enqueued first, each into its own output, and only then checked: sampled rows of every call
against the fp64 oracle, the buffer against the last step, the device status word (a bounded
wait that gave up would show as PF_ERR_TIMEOUT), the key-range split's counters, which must
all be back at zero, and the per-layer ordering counters.
"""
import numpy as np
import pytest
import torch

import oracle
import patch_attention_b200 as pa
from patch_attention_b200 import synth
from tests._oracle_util import f64

pytestmark = pytest.mark.gpu

PF, DF, PF2 = pa.PF_SCHED_PIPEFUSION, pa.PF_SCHED_DISTRIFUSION, pa.PF_SCHED_PIPEFUSION_2H


@pytest.mark.parametrize("d,schedule,B", [(64, PF, 1), (72, PF, 1), (128, PF, 1), (64, DF, 1), (128, DF, 1),
                                          (72, PF, 2), (64, PF2, 1), (72, PF2, 1), (128, PF2, 1),
                                          (72, PF2, 2)])
def test_overlapped_micro_steps_match_the_oracle(d, schedule, B):
    wl = synth.AttnWorkload("b2b", batch=B, heads=4, head_dim=d, grid_h=64, grid_w=64,
                            n_patches=8, n_txt=77, n_layers=2, n_steps=3, ar_a=0.95, ar_b=0.3)
    S, L, M, P, T = wl.n_steps, wl.n_layers, wl.n_patches, wl.patch_len, wl.n_txt
    gen = synth.AttnInputs(wl, seed=21, device="cuda")
    steps = [[gen.step_tensors(l) for l in range(L)] for _ in range(S)]
    g = torch.Generator(device="cuda").manual_seed(5)
    q_txt = [torch.randn(B, T, wl.heads, d, device="cuda", generator=g).bfloat16() for _ in range(L)]
    pat = pa.PatchAttention(B, wl.heads, d, wl.n_img, M, T, L, schedule=schedule)
    outs, txt_outs, mid_outs = {}, {}, {}
    try:
        for l in range(L):
            pat.init_layer(l, steps[0][l]["k"], steps[0][l]["v"])
        patches = [[[(t["q"][:, p * P:(p + 1) * P].contiguous(), t["k"][:, p * P:(p + 1) * P].contiguous(),
                      t["v"][:, p * P:(p + 1) * P].contiguous()) for p in range(M)] for t in st] for st in steps]
        torch.cuda.synchronize()
        # every call of every step, in the pipeline's order, without a synchronisation
        for s in range(S):
            for p in range(M):
                for l in range(L):
                    q, k, v = patches[s][l][p]
                    t = steps[s][l]
                    outs[(s, l, p)] = pat.step(l, p, q, k, v, t["k_txt"], t["v_txt"])
                if p == 1:
                    # text queries in the middle of the step: the buffer as it stands
                    for l in range(L):
                        t = steps[s][l]
                        mid_outs[(s, l)] = pat.text_step(l, q_txt[l], t["k_txt"], t["v_txt"])
            for l in range(L):
                t = steps[s][l]
                txt_outs[(s, l)] = pat.text_step(l, q_txt[l], t["k_txt"], t["v_txt"])
        torch.cuda.synchronize()
        pat.check()  # no bounded wait gave up
        rng = np.random.default_rng(3)
        attention = oracle.distrifusion_attention if schedule == DF else oracle.patch_attention
        for (s, l, p), o in outs.items():
            cur, prev = steps[s][l], steps[max(s - 1, 0)][l]
            rows = sorted(set([0, P - 1] + list(rng.integers(0, P, 6))))
            h, bi = int(rng.integers(0, wl.heads)), int(rng.integers(0, B))
            take = lambda x: f64(x[bi][:, h:h + 1])
            ref = attention(take(cur["q"]), take(cur["k"]), take(cur["v"]), take(prev["k"]),
                            take(prev["v"]), take(cur["k_txt"]), take(cur["v_txt"]), p, M,
                            wl.softmax_scale, rows=rows)
            got = f64(o[bi][rows][:, h:h + 1])
            rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
            assert rel <= 5e-3, (s, l, p, rel)
        for (s, l), o in txt_outs.items():
            # after a step's last patch the buffer holds that step's K/V under both schedules
            cur = steps[s][l]
            h, bi = int(rng.integers(0, wl.heads)), int(rng.integers(0, B))
            rows = sorted(set([0, T - 1] + list(rng.integers(0, T, 6))))
            take = lambda x: f64(x[bi][:, h:h + 1])
            ref = oracle.attend(take(q_txt[l])[rows], np.concatenate([take(cur["k"]), take(cur["k_txt"])]),
                                np.concatenate([take(cur["v"]), take(cur["v_txt"])]), wl.softmax_scale)
            got = f64(o[bi][rows][:, h:h + 1])
            rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
            assert rel <= 5e-3, (s, l, "text", rel)
        for (s, l), o in mid_outs.items():
            # after patch 1: this step's rows for patches 0-1 and the previous step's for the
            # rest under PipeFusion (either layout); the previous step everywhere under
            # DistriFusion
            cur, prev = steps[s][l], steps[max(s - 1, 0)][l]
            h, bi = int(rng.integers(0, wl.heads)), int(rng.integers(0, B))
            rows = sorted(set([0, T - 1] + list(rng.integers(0, T, 6))))
            take = lambda x: f64(x[bi][:, h:h + 1])
            if schedule == DF:
                kb, vb = take(prev["k"]), take(prev["v"])
            else:
                kb = oracle.expected_buffer(take(cur["k"]), take(prev["k"]), 1, M)
                vb = oracle.expected_buffer(take(cur["v"]), take(prev["v"]), 1, M)
            ref = oracle.attend(take(q_txt[l])[rows], np.concatenate([kb, take(cur["k_txt"])]),
                                np.concatenate([vb, take(cur["v_txt"])]), wl.softmax_scale)
            got = f64(o[bi][rows][:, h:h + 1])
            rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
            assert rel <= 5e-3, (s, l, "mid-step text", rel)
        for l in range(L):
            # after the step's last patch the half being read holds the step
            last_k, last_v = steps[-1][l]["k"].view(torch.int16), steps[-1][l]["v"].view(torch.int16)
            kb, vb = pat.buffer_kv(l, pat.read_half(l))
            assert torch.equal(kb.view(torch.int16), last_k) and torch.equal(vb.view(torch.int16), last_v), l
        # between launches every split counter (parts arrived, partials written: two per query
        # tile of every pair) is back at 0, the merger of each query tile resets them; the
        # per-layer ordering counters that follow them count, for every CTA of a patch call,
        # one finished scatter, and for every CTA of every call one finished read of the
        # buffer: every word before them is zero, and they are one (scatter, read) pair of
        # non-zero counts per layer with more reads than scatters (partial slots follow)
        assert pat.workspace is not None
        words = pat.workspace[:4096].view(torch.int64)
        first = int(torch.nonzero(words).flatten()[0])
        assert first % 2 == 0 and first >= 2, first
        order = words[first:first + 2 * L].view(L, 2)
        assert bool((order > 0).all()) and bool((order[:, 1] > order[:, 0]).all()), order
    finally:
        pat.close()


@pytest.mark.parametrize("schedule", [PF, PF2])
def test_workspace_detached_and_attached_between_steps(schedule):
    """Calls without a workspace wait for the previous grid; attaching a workspace again zeroes
    the counters (ordered after the calls still running on the stream) and restarts the host's
    targets.  Steps alternate between the two, still without host synchronisation."""
    d = 128
    wl = synth.AttnWorkload("b2bws", batch=1, heads=2, head_dim=d, grid_h=32, grid_w=64,
                            n_patches=4, n_txt=33, n_layers=2, n_steps=4, ar_a=0.95, ar_b=0.3)
    S, L, M, P = wl.n_steps, wl.n_layers, wl.n_patches, wl.patch_len
    gen = synth.AttnInputs(wl, seed=8, device="cuda")
    steps = [[gen.step_tensors(l) for l in range(L)] for _ in range(S)]
    pat = pa.PatchAttention(1, wl.heads, d, wl.n_img, M, wl.n_txt, L, schedule=schedule)
    ws = pat.workspace
    assert ws is not None
    outs = {}
    try:
        for l in range(L):
            pat.init_layer(l, steps[0][l]["k"], steps[0][l]["v"])
        for s in range(S):
            pa.pf_set_workspace(pat.ctx, ws if s % 2 == 0 else None)
            for p in range(M):
                for l in range(L):
                    t = steps[s][l]
                    sl = slice(p * P, (p + 1) * P)
                    outs[(s, l, p)] = pat.step(l, p, t["q"][:, sl].contiguous(), t["k"][:, sl].contiguous(),
                                               t["v"][:, sl].contiguous(), t["k_txt"], t["v_txt"])
        torch.cuda.synchronize()
        pat.check()
        rng = np.random.default_rng(4)
        for (s, l, p), o in outs.items():
            cur, prev = steps[s][l], steps[max(s - 1, 0)][l]
            rows = sorted(set([0, P - 1] + list(rng.integers(0, P, 6))))
            h = int(rng.integers(0, wl.heads))
            take = lambda x: f64(x[0][:, h:h + 1])
            ref = oracle.patch_attention(take(cur["q"]), take(cur["k"]), take(cur["v"]), take(prev["k"]),
                                         take(prev["v"]), take(cur["k_txt"]), take(cur["v_txt"]), p, M,
                                         wl.softmax_scale, rows=rows)
            got = f64(o[0][rows][:, h:h + 1])
            rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
            assert rel <= 5e-3, (s, l, p, rel)
        for l in range(L):
            kb, vb = pat.buffer_kv(l, pat.read_half(l))
            assert torch.equal(kb.view(torch.int16), steps[-1][l]["k"].view(torch.int16))
            assert torch.equal(vb.view(torch.int16), steps[-1][l]["v"].view(torch.int16))
    finally:
        pat.close()

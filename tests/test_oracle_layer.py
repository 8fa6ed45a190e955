"""Layer-level pins for the oracle.

* The authors' blog post ("硬件高效實現", hardware-efficient implementation)
  states that running each memory's operator separately and summing the
  router-weighted outputs equals mixing the memories first and reading the
  mixture out: checked between two independently written forms.
* One memory with top-1 reduces the layer to two plain Gated DeltaNets (the
  shared memory and memory 0) summed.
* Sequences in a packed batch are independent; a state handed from one call
  to the next continues the recurrence; decode continues a prefill
  (constant-cost inference: the blog post's introduction and the paper
  card's Summary).
* A memory neither decays nor updates on tokens not routed to it.
"""
import numpy as np
import pytest

from mixture_memories_layer_b200 import synth
from oracle import mom_oracle as orc


def _tiny(seed=0, N=None, M=4, k=2, H=2, d=8, D=16, varlen=False):
    w = synth.Workload("t", 1, N or 24, D, H, d, M, k, "f32", seed=seed)
    rng = np.random.default_rng(seed)
    p = synth.make_weights(w, rng)
    if varlen:
        cu = np.array([0, 9, 9, 20, 31], dtype=np.int32)
    else:
        cu = np.array([0, w.seq_len], dtype=np.int32)
    x = synth.make_tokens(w, rng, int(cu[-1]))
    return w, p, x, cu


@pytest.mark.parametrize("varlen", [False, True])
def test_mixed_state_equals_output_sum(varlen):
    w, p, x, cu = _tiny(seed=1, varlen=varlen)
    r = orc.mom_forward(x, p, cu, w.top_k, w.heads, w.d_head, scale=1.0)
    mixed = orc.mom_forward_mixed_state(x, p, cu, w.top_k, w.heads, w.d_head, scale=1.0)
    assert np.allclose(r["out"], mixed, rtol=0, atol=1e-12)


def test_one_memory_top1_is_two_plain_gdns():
    w, p, x, cu = _tiny(seed=2, M=1, k=1)
    r = orc.mom_forward(x, p, cu, 1, w.heads, w.d_head)
    assert np.all(r["idx"] == 0) and np.allclose(r["gate"], 1.0)
    q, k_sh, v_sh, b, la = orc.shared_projections(x, p, w.heads, w.d_head)
    k0, v0 = orc.memory_kv(x, p, 0, w.heads, w.d_head)
    o_sh, _ = orc.gdn_chunked(q, k_sh, v_sh, b, la, chunk=5)
    o_0, S0 = orc.gdn_chunked(q, k0, v0, b, la, chunk=5)
    assert np.allclose(r["out"], o_sh + o_0, atol=1e-11)
    assert np.allclose(r["h_mem"][0, 0], S0, atol=1e-11)


def test_packed_sequences_are_independent():
    w, p, x, cu = _tiny(seed=3, varlen=True)
    r = orc.mom_forward(x, p, cu, w.top_k, w.heads, w.d_head)
    for s in range(len(cu) - 1):
        t0, t1 = cu[s], cu[s + 1]
        one = orc.mom_forward(x[t0:t1], p, np.array([0, t1 - t0]), w.top_k, w.heads, w.d_head)
        assert np.allclose(r["out"][t0:t1], one["out"], atol=1e-13)
        assert np.allclose(r["h_shared"][s], one["h_shared"][0], atol=1e-13)
        assert np.allclose(r["h_mem"][:, s], one["h_mem"][:, 0], atol=1e-13)


def test_state_hand_off_between_calls():
    w, p, x, cu = _tiny(seed=4, N=30)
    full = orc.mom_forward(x, p, cu, w.top_k, w.heads, w.d_head)
    a = orc.mom_forward(x[:13], p, np.array([0, 13]), w.top_k, w.heads, w.d_head)
    b = orc.mom_forward(x[13:], p, np.array([0, 17]), w.top_k, w.heads, w.d_head,
                        h0_shared=a["h_shared"], h0_mem=a["h_mem"])
    assert np.allclose(np.concatenate([a["out"], b["out"]]), full["out"], atol=1e-12)
    assert np.allclose(b["h_mem"], full["h_mem"], atol=1e-12)
    assert np.allclose(b["h_shared"], full["h_shared"], atol=1e-12)


def test_decode_continues_prefill():
    w, p, x, cu = _tiny(seed=5, N=21)
    B = 3
    # three sequences: prefill of 20 tokens each, then one decode token each
    rng = np.random.default_rng(50)
    xs = synth.make_tokens(w, rng, B * 21).reshape(B, 21, -1)
    pre = orc.mom_forward(xs[:, :20].reshape(B * 20, -1), p, np.arange(0, B * 20 + 1, 20),
                          w.top_k, w.heads, w.d_head, scale=0.9)
    state = orc.decode_state_from_prefill(pre["h_shared"], pre["h_mem"])
    out, new, idx, gate, _ = orc.mom_decode_step(xs[:, 20], p, state, w.top_k, w.heads, w.d_head, scale=0.9)
    full = orc.mom_forward(xs.reshape(B * 21, -1), p, np.arange(0, B * 21 + 1, 21),
                           w.top_k, w.heads, w.d_head, scale=0.9)
    assert np.allclose(out, full["out"][20::21], atol=1e-12)
    ref_state = orc.decode_state_from_prefill(full["h_shared"], full["h_mem"])
    assert np.allclose(new, ref_state, atol=1e-12)


def test_unrouted_memory_is_frozen():
    w, p, x, cu = _tiny(seed=6, N=20)
    r = orc.mom_forward(x, p, cu, w.top_k, w.heads, w.d_head)
    forced = r["idx"].copy()
    # memory 3 sees only tokens 0..4; afterwards route those slots elsewhere
    for t in range(20):
        if t >= 5 and 3 in forced[t]:
            forced[t][list(forced[t]).index(3)] = [m for m in range(3) if m not in forced[t]][0]
    f = orc.mom_forward(x, p, cu, w.top_k, w.heads, w.d_head, forced_idx=forced)
    head = orc.mom_forward(x[:5], p, np.array([0, 5]), w.top_k, w.heads, w.d_head, forced_idx=forced[:5])
    assert np.allclose(f["h_mem"][3, 0], head["h_mem"][3, 0], atol=1e-13)
    assert not np.allclose(f["h_mem"][3, 0], 0.0)


def test_forced_routing_equal_to_natural_changes_nothing():
    w, p, x, cu = _tiny(seed=7)
    r = orc.mom_forward(x, p, cu, w.top_k, w.heads, w.d_head)
    f = orc.mom_forward(x, p, cu, w.top_k, w.heads, w.d_head, forced_idx=r["idx"])
    assert np.array_equal(r["out"], f["out"]) and np.array_equal(r["gate"], f["gate"])


def test_permuted_rows_reproduce_memory_outputs():
    """Running each (memory, sequence) segment of the reordered rows through
    the recurrence reproduces o_mem: the reordering loses nothing."""
    w, p, x, cu = _tiny(seed=8, varlen=True)
    r = orc.mom_forward(x, p, cu, w.top_k, w.heads, w.d_head)
    perm, row_of, offs, seg = orc.permute(r["idx"], w.n_mem, cu)
    S = len(cu) - 1
    o_rows = np.zeros((len(perm), w.heads, w.d_head))
    for m in range(w.n_mem):
        for s in range(S):
            a, b = seg[m * S + s], seg[m * S + s + 1]
            toks = perm[a:b]
            if len(toks) == 0:
                continue
            km, vm = orc.memory_kv(x[toks], p, m, w.heads, w.d_head)
            o_rows[a:b], _ = orc.gdn_recurrence(r["q"][toks], km, vm, r["beta"][toks], r["log_alpha"][toks])
    k = w.top_k
    for t in range(len(x)):
        for j in range(k):
            assert np.allclose(o_rows[row_of[t * k + j]], r["o_mem"][t, j], atol=1e-13)

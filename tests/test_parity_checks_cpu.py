"""The GPU parity checkers themselves, on the CPU: fed the oracle's own stage values as if a kernel
had produced them, they pass; fed a corrupted stage, a code off by one away from a near-tie, or a
wrong residual, they fail; and the near-tie rule (both sides decide in float32) marks
exactly the rows it should. A checker that accepted anything would make every GPU parity test
vacuous."""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from parity_checks import _codes_match, chain_clean_rows, check_block_stages, oracle_chain_groups


def _oracle_taps(x, qp, h0=None):
    """Every stage of one block as the kernel's debug taps would hold it, computed by the oracle."""
    B, T, d = x.shape
    m = B * T
    x2 = x.reshape(m, d).astype(np.float64)
    q_ifg, deq_ifg, z = [], [], []
    for p in ("i", "f", "g"):
        y, tp = O.bitlinear(x2, qp[f"nw_{p}"], qp[f"t_{p}"], qp[f"s_{p}"])
        q_ifg.append(tp["q"])
        deq_ifg.append(tp["deq"])
        z.append(y)
    zi, zf, g = z
    f, i = O.hgrn_gates(zf.reshape(B, T, d), zi.reshape(B, T, d))
    h = O.hgrn_scan(f, i, h0)
    u = O.rmsnorm(h.reshape(m, d), qp["gnorm_w"]) * O.silu(g)
    o, to = O.bitlinear(u, qp["nw_o"], qp["t_o"], qp["s_o"])
    x1 = x2 + o
    gu, tg = O.bitlinear(x1, qp["nw_gate"], qp["t_gate"], qp["s_gate"])
    inner = gu.shape[1] // 2
    v = O.silu(gu[:, :inner]) * gu[:, inner:]
    dn, td = O.bitlinear(v, qp["nw_down"], qp["t_down"], qp["s_down"])
    y = x1 + dn
    T32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    I8 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int8))
    taps = {"q_ifg": I8(np.stack(q_ifg)), "deq_ifg": T32(np.stack(deq_ifg)), "z": T32(np.concatenate(z, 1)),
            "h": T32(h.reshape(m, d)), "q_o": I8(to["q"]), "deq_o": T32(to["deq"]), "x1": T32(x1),
            "q_gate": I8(tg["q"]), "deq_gate": T32(tg["deq"]), "gu": T32(gu), "v": T32(v),
            "q_down": I8(td["q"]), "deq_down": T32(td["deq"])}
    return taps, y.reshape(B, T, d), h[:, -1]


@pytest.fixture(scope="module")
def case():
    sh = synth.BlockShape("t", 32, 64, 1)
    qp = O.quantize_block(synth.block_params(300, sh, random_norms=True))
    x = synth.activations(301, (2, 9, 32))
    h0 = synth.activations(302, (2, 32)) * 0.5
    taps, y, hl = _oracle_taps(x, qp, h0)
    return x, qp, h0, taps, y, hl


def _check(case, taps=None, y=None, glu_fused=False):
    x, qp, h0, t0, y0, hl = case
    check_block_stages(x, qp, taps if taps is not None else t0, y if y is not None else y0, hl, h0, bf16=False,
                       glu_fused=glu_fused)


def test_stage_checker_accepts_the_oracles_own_stages(case):
    _check(case)
    _check(case, glu_fused=True)


@pytest.mark.parametrize("stage", ["z", "h", "x1", "gu", "v", "deq_o", "y"])
def test_stage_checker_rejects_a_corrupted_float_stage(case, stage):
    x, qp, h0, taps, y, hl = case
    bad = dict(taps)
    if stage == "y":
        y = y.copy()
        y[1, 4, 7] += 0.05 * (1 + abs(y[1, 4, 7]))
    else:
        t = taps[stage].clone()
        t.view(-1)[t.numel() // 3] *= 1.05
        t.view(-1)[t.numel() // 3] += 1e-3
        bad[stage] = t
    with pytest.raises(AssertionError):
        _check(case, taps=bad, y=y, glu_fused=stage == "v")


@pytest.mark.parametrize("stage", ["q_ifg", "q_o", "q_gate", "q_down"])
def test_stage_checker_rejects_a_code_off_by_one_away_from_a_tie(case, stage):
    x, qp, h0, taps, y, hl = case
    bad = dict(taps)
    q = taps[stage].clone()
    flat = q.view(-1)
    j = int(np.argmin(np.abs(flat.numpy().astype(int))))       # a small code, far from the clamp
    flat[j] += 1
    bad[stage] = q
    with pytest.raises(AssertionError):
        _check(case, taps=bad)


def test_code_rule_allows_one_step_only_at_a_near_tie():
    v = np.array([[0.50004, 1.2, -3.49996, 2.0]], dtype=np.float32)
    q_ref = np.rint(v).astype(np.int8)                           # [1, 1, -3, 2]
    assert q_ref.tolist() == [[1, 1, -3, 2]]
    _codes_match(np.array([[0, 1, -4, 2]], np.int8), v, q_ref, 1e-4)   # both flips sit at ties
    with pytest.raises(AssertionError):
        _codes_match(np.array([[1, 2, -3, 2]], np.int8), v, q_ref, 1e-4)   # 1.2 is no tie
    with pytest.raises(AssertionError):
        _codes_match(np.array([[-1, 1, -3, 2]], np.int8), v, q_ref, 1e-4)  # two steps at a tie


def test_chain_rule_marks_rows_after_a_tie_and_rejects_other_flips():
    B, T, k = 1, 4, 3
    v = np.array([[0.2, 1.1, -2.3], [0.50002, 4.0, 1.0], [3.2, 1.0, 1.0], [0.1, 0.1, 0.1]], np.float32)
    q = np.rint(v).astype(np.int8)
    flipped = q.copy()
    assert q[1, 0] == 1
    flipped[1, 0] = 0                                            # row 1: a flip at a near-tie
    groups_o = [[(q, v)]]
    # outside the recurrence only the flipped row is dirty; through it, every later step too
    assert chain_clean_rows([[flipped]], groups_o, B, T, scan_groups=set(), margins=[1e-4]).tolist() == \
        [True, False, True, True]
    assert chain_clean_rows([[flipped]], groups_o, B, T, scan_groups={0}, margins=[1e-4]).tolist() == \
        [True, False, False, False]
    off = q.copy()
    off[2, 0] = 4                                                # 3.2 -> 4: not a tie
    with pytest.raises(AssertionError):
        chain_clean_rows([[off]], groups_o, B, T, scan_groups=set(), margins=[1e-4])
    # a later group may differ anywhere in a row that is already dirty
    later_v = np.full((T, k), 0.2, np.float32)
    later_q = np.rint(later_v).astype(np.int8)
    later_k = later_q.copy()
    later_k[3, 1] = 1                                            # row 3, far from a tie
    clean = chain_clean_rows([[flipped], [later_k]], [[(q, v)], [(later_q, later_v)]], B, T,
                             scan_groups={0}, margins=[1e-4, 1e-3])
    assert clean.tolist() == [True, False, False, False]


def test_oracle_chain_groups_follow_the_block(case):
    x, qp, h0, taps, y, hl = case
    y_ref, _, inter = O.block_forward(x.astype(np.float64), qp)
    groups = oracle_chain_groups(x.astype(np.float64), qp, inter)
    assert [len(g) for g in groups] == [3, 1, 1, 1]
    q_i, _ = groups[0][0]
    assert np.array_equal(q_i, taps["q_ifg"][0].numpy())


def test_chain_checker_over_two_layers():
    from parity_checks import check_chain_end_to_end

    sh = synth.BlockShape("t", 32, 64, 1)
    qps = [O.quantize_block(synth.block_params(310 + l, sh, random_norms=True)) for l in range(2)]
    x = synth.activations(312, (2, 5, 32))
    taps, states, cur = [], [], x.astype(np.float64)
    for qp in qps:
        t, y, hl = _oracle_taps(cur, qp)
        taps.append(t)
        states.append(hl)
        cur = y
    rel, clean = check_chain_end_to_end(x, qps, taps, cur, states_g=states)
    assert rel < 1e-12 and clean == 1.0
    bad = cur.copy()
    bad[0, 2, 5] += 1e-2 * (1 + abs(bad[0, 2, 5]))
    with pytest.raises(AssertionError):
        check_chain_end_to_end(x, qps, taps, bad, states_g=states)
    bad_states = [s.copy() for s in states]
    bad_states[1][1, 3] += 1e-2
    with pytest.raises(AssertionError):
        check_chain_end_to_end(x, qps, taps, cur, states_g=bad_states)

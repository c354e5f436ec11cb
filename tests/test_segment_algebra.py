"""The sequence split of the inner-product rule (Falcon-1A), checked on the CPU against
the fp64 oracle.

The additive write S_t = alpha_t S_{t-1} + beta_t y_t x_t^T ("Fast Weight Attention for
Continual Learning", authors' abstract) has a scalar transition, so a run of tokens maps
S to 2^(G_end) S + D with D = sum_t 2^(G_end - G_t) beta_t y_t x_t^T (G the cumulative
log2 decay of the run). The CUDA path computes D per piece in parallel, scans the pieces
into the state at each segment start, and runs every segment as a head of its own from
that state and the key cached before it. This restates those three steps in numpy (fp64)
and requires the concatenated segment outputs and the final state to equal one oracle
pass over the whole sequence.
"""
import numpy as np
import pytest

import oracle
from delta_rule_linear_falcon_b200 import inputs as I

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def piece_increment(x, y, alpha, eta, eps):
    """D and G_end of one run of pairs (x_t, y_t), positive-decay form."""
    alpha, eta = alpha.astype(np.float64), eta.astype(np.float64)
    G = np.cumsum(np.log2(alpha))
    nrm = np.einsum("td,td->t", x, x)
    den = nrm + eps
    beta = np.where(den > 0, eta / np.where(den > 0, den, 1.0), 0.0)
    w = beta * np.exp2(np.minimum(G[-1] - G, 0.0))
    return (w[:, None] * y).T @ x, G[-1]


def split_forward(s: I.SeqInputs, nseg: int, piece: int, same_step: bool, check_final: bool = True):
    B, H, T, dk = s.k.shape
    dv = s.v.shape[-1]
    L = T // nseg
    o = np.zeros((B, H, T, dv))
    S_fin = np.zeros((B, H, dv, dk))
    for b in range(B):
        for h in range(H):
            k, v = s.k[b, h].astype(np.float64), s.v[b, h].astype(np.float64)
            kp = s.k_prev[b, h].astype(np.float64) if s.k_prev is not None else np.zeros(dk)
            x = k if same_step else np.concatenate([kp[None], k[:-1]], axis=0)
            S = s.S0[b, h].astype(np.float64) if s.S0 is not None else np.zeros((dv, dk))
            starts = []
            for sg in range(nseg):
                starts.append(S.copy())
                for p0 in range(sg * L, (sg + 1) * L, piece):
                    sl = slice(p0, p0 + piece)
                    D, g = piece_increment(x[sl], v[sl], s.alpha[b, h, sl], s.eta[b, h, sl], s.eps)
                    S = np.exp2(min(g, 0.0)) * S + D
            S_fin[b, h] = S
            for sg in range(nseg):
                sl = slice(sg * L, (sg + 1) * L)
                if same_step:
                    kprev_seg = None
                elif sg == 0:
                    kprev_seg = s.k_prev[b, h] if s.k_prev is not None else None
                else:
                    kprev_seg = k[sg * L - 1]
                o_s, S_s, _ = oracle.recurrent(
                    s.rule, s.q[b, h, sl][None, None], s.k[b, h, sl][None, None], s.v[b, h, sl][None, None],
                    s.alpha[b, h, sl][None, None], s.eta[b, h, sl][None, None], s.eps,
                    S0=starts[sg][None, None],
                    k_prev=None if kprev_seg is None else kprev_seg[None, None])
                o[b, h, sl] = o_s[0, 0]
                if check_final and sg == nseg - 1:
                    # the last segment's own pass and the scan agree on the final state
                    assert np.allclose(S_s[0, 0], S, rtol=1e-10, atol=1e-12)
    return o, S_fin


@pytest.mark.parametrize("nseg,piece", [(2, 64), (4, 32), (3, 48), (6, 8)])
@pytest.mark.parametrize("same_step", [False, True])
def test_split_equals_one_pass(nseg, piece, same_step):
    T = 96 * nseg if nseg != 6 else 144
    rule = 2 | (0x100 if same_step else 0)
    s = I.make_seq(rule, 1, 2, T - T % (nseg * piece), 8, 6, seed=900 + nseg, io_dtype="f32",
                   with_state=True, with_kprev=True, alpha_mu=1.0)
    o_ref, S_ref, _ = oracle.recurrent(s.rule, s.q, s.k, s.v, s.alpha, s.eta, s.eps, S0=s.S0, k_prev=s.k_prev)
    o, S = split_forward(s, nseg, piece, same_step)
    assert np.max(np.abs(o - o_ref)) <= 1e-11 * max(1.0, np.max(np.abs(o_ref)))
    assert np.max(np.abs(S - S_ref)) <= 1e-11 * max(1.0, np.max(np.abs(S_ref)))


def test_split_without_cached_key_or_state():
    s = I.make_seq(2, 2, 1, 128, 8, 8, seed=910, io_dtype="f32")
    o_ref, S_ref, _ = oracle.recurrent(s.rule, s.q, s.k, s.v, s.alpha, s.eta, s.eps)
    o, S = split_forward(s, 4, 16, False)
    assert np.max(np.abs(o - o_ref)) <= 1e-11 * np.max(np.abs(o_ref))
    assert np.max(np.abs(S - S_ref)) <= 1e-11 * np.max(np.abs(S_ref))


def test_split_is_wrong_for_the_regression_rule():
    """The split relies on the additive write: the same steps applied to Falcon-1, whose
    transition alpha (I - beta x x^T) depends on the keys, must not reproduce the oracle."""
    s = I.make_seq(1, 1, 1, 128, 8, 8, seed=920, io_dtype="f32", with_state=True, alpha_mu=1.0)
    o_ref, _, _ = oracle.recurrent(1, s.q, s.k, s.v, s.alpha, s.eta, s.eps, S0=s.S0)
    s2 = I.SeqInputs(**{**s.__dict__, "rule": 1})
    o, _ = split_forward(s2, 2, 64, False, check_final=False)
    assert np.max(np.abs(o - o_ref)) > 1e-3 * np.max(np.abs(o_ref))

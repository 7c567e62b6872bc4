"""Pins for the fp64 oracle: checks against things other than the oracle itself.

The pages ("M²RNN: Non-Linear RNNs with Matrix-Valued States for Scalable
Language Modeling", gist.science technical summary §2.1) fix only the two
state-update equations, the shapes and the gate's range; they print no worked
example.  So the oracle is pinned by:
  * closed forms of special cases (W = 0 and f = 0; f = 1; W = 0, constant f),
  * a library routine: with f = 0 every row of H is an Elman tanh RNN, which
    torch.nn.RNN evaluates (forward and autograd) in fp64,
  * invariants: convex-blend bound, row/column permutation equivariance,
    batch and head independence, thread-count independence,
  * a 2×2 case written out scalar by scalar,
  * central finite differences of the oracle's own forward for every input
    of the backward, plus backward closed forms for f = 1 and for W = 0, f = 0.
Each check is chosen so that a plausible slip (transposed W, wrong gate
direction, readout before the update, dropped rank-1 term, off-by-one in the
BPTT) fails at least one of them.
"""
import numpy as np
import pytest
import torch

from oracle import oracle


def _rand(B=2, H=3, T=7, K=4, V=5, seed=0, scale=0.7, h0=True):
    r = np.random.default_rng(seed)
    k = r.standard_normal((B, H, T, K)) * scale
    v = r.standard_normal((B, H, T, V)) * scale
    q = r.standard_normal((B, H, T, K)) * scale
    f = 1.0 / (1.0 + np.exp(-r.standard_normal((B, H, T)) - 1.0))
    W = r.standard_normal((H, V, V)) * (1.5 / np.sqrt(V))
    H0 = r.uniform(-0.9, 0.9, (B, H, K, V)) if h0 else None
    return k, v, q, f, W, H0


def test_closed_form_W0_f0():
    # W = 0, f = 0  =>  H_t = tanh(k_t v_tᵀ), y_t = H_tᵀ q_t  (from the §2.1 equations)
    k, v, q, f, W, H0 = _rand()
    W[:] = 0.0
    f[:] = 0.0
    y, HT = oracle.forward(k, v, q, f, W, H0)
    Ht = np.tanh(np.einsum("bhti,bhtj->bhtij", k, v))
    np.testing.assert_allclose(y, np.einsum("bhtij,bhti->bhtj", Ht, q), rtol=0, atol=1e-14)
    np.testing.assert_allclose(HT, Ht[:, :, -1], rtol=0, atol=1e-15)


def test_f1_keeps_initial_state():
    # f = 1  =>  H_t = H0 for all t, y_t = H0ᵀ q_t
    k, v, q, f, W, H0 = _rand()
    f[:] = 1.0
    y, HT = oracle.forward(k, v, q, f, W, H0)
    np.testing.assert_array_equal(HT, H0)
    np.testing.assert_allclose(y, np.einsum("bhij,bhti->bhtj", H0, q), rtol=0, atol=1e-14)


def test_ema_closed_form_W0_constant_gate():
    # W = 0, f_t = c  =>  H_T = c^T H0 + sum_s (1-c) c^(T-1-s) tanh(k_s v_sᵀ)
    k, v, q, f, W, H0 = _rand(T=9)
    W[:] = 0.0
    c = 0.63
    f[:] = c
    _, HT = oracle.forward(k, v, q, f, W, H0)
    T = k.shape[2]
    ref = c ** T * H0
    for s in range(T):
        ref = ref + (1 - c) * c ** (T - 1 - s) * np.tanh(np.einsum("bhi,bhj->bhij", k[:, :, s], v[:, :, s]))
    np.testing.assert_allclose(HT, ref, rtol=0, atol=1e-14)


def _torch_rnn_rows(k, v, W, H0):
    """Each row i of H with f = 0 is h_t = tanh(x_t + Wᵀ h_{t-1}) with x_t = k_t[i] v_t.

    torch.nn.RNN computes h_t = tanh(W_ih x_t + W_hh h_{t-1}); we set W_ih = I and
    W_hh = Wᵀ (so that the row vector update is h_tᵀ = tanh(x_tᵀ + h_{t-1}ᵀ W)).
    Returns the RNN module and the per-row outputs [B,H,K,T,V].
    """
    B, Hh, T, K = k.shape
    V = v.shape[-1]
    outs = []
    mods = []
    for h in range(Hh):
        rnn = torch.nn.RNN(input_size=V, hidden_size=V, num_layers=1, nonlinearity="tanh",
                           bias=False, batch_first=True).double()
        with torch.no_grad():
            rnn.weight_ih_l0.copy_(torch.eye(V, dtype=torch.float64))
            rnn.weight_hh_l0.copy_(torch.from_numpy(W[h].T.copy()))
        # sequences: one per (b, i): input k[b,h,t,i] * v[b,h,t,:]
        x = torch.from_numpy(np.einsum("bti,btj->bitj", k[:, h], v[:, h]).reshape(B * K, T, V).copy())
        h0 = torch.from_numpy(H0[:, h].reshape(B * K, V).copy()).unsqueeze(0)
        x.requires_grad_(True)
        h0.requires_grad_(True)
        out, _ = rnn(x, h0)
        outs.append((out, x, h0))
        mods.append(rnn)
    return mods, outs


def test_f0_rows_are_torch_elman_rnns():
    k, v, q, f, W, H0 = _rand(B=2, H=2, T=6, K=3, V=4, seed=3)
    f[:] = 0.0
    y, HT = oracle.forward(k, v, q, f, W, H0)
    B, Hh, T, K = k.shape
    V = v.shape[-1]
    _, outs = _torch_rnn_rows(k, v, W, H0)
    for h in range(Hh):
        out = outs[h][0].detach().numpy().reshape(B, K, T, V)      # H_t rows
        np.testing.assert_allclose(HT[:, h], out[:, :, -1], rtol=0, atol=1e-13)
        y_ref = np.einsum("bitj,bti->btj", out, q[:, h])
        np.testing.assert_allclose(y[:, h], y_ref, rtol=0, atol=1e-13)


def test_f0_backward_matches_torch_autograd():
    k, v, q, f, W, H0 = _rand(B=2, H=2, T=5, K=3, V=4, seed=4)
    f[:] = 0.0
    r = np.random.default_rng(9)
    dy = r.standard_normal((2, 2, 5, 4))
    dHT = r.standard_normal((2, 2, 3, 4))
    g = oracle.backward(k, v, q, f, W, H0, dy, dHT)
    B, Hh, T, K = k.shape
    V = v.shape[-1]
    mods, outs = _torch_rnn_rows(k, v, W, H0)
    for h in range(Hh):
        out, x, h0 = outs[h]
        o = out.reshape(B, K, T, V)
        y = torch.einsum("bitj,bti->btj", o, torch.from_numpy(q[:, h].copy()))
        loss = (y * torch.from_numpy(dy[:, h].copy())).sum() + (o[:, :, -1] * torch.from_numpy(dHT[:, h].copy())).sum()
        loss.backward()
        # dW: weight_hh = Wᵀ
        np.testing.assert_allclose(g["dW"][h], mods[h].weight_hh_l0.grad.numpy().T, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(g["dH0"][:, h], h0.grad.numpy().reshape(B, K, V), rtol=1e-10, atol=1e-12)
        # input x[b*K+i, t, :] = k[b,h,t,i] v[b,h,t,:]; chain rule to k and v
        gx = x.grad.numpy().reshape(B, K, T, V)
        dk = np.einsum("bitj,btj->bti", gx, v[:, h])
        dv = np.einsum("bitj,bti->btj", gx, k[:, h])
        np.testing.assert_allclose(g["dk"][:, h], dk, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(g["dv"][:, h], dv, rtol=1e-10, atol=1e-12)


def test_convex_blend_bound():
    # |H0| <= 1 elementwise  =>  |H_t| <= 1 for every t (H_t is a convex blend of H_{t-1} and a tanh)
    k, v, q, f, W, H0 = _rand(B=1, H=2, T=40, K=5, V=6, seed=5, scale=3.0)
    W *= 4.0
    H0 = np.clip(H0 / 0.9, -1.0, 1.0)
    for T in (1, 2, 5, 17, 40):
        _, HT = oracle.forward(k[:, :, :T], v[:, :, :T], q[:, :, :T], f[:, :, :T], W, H0)
        assert np.abs(HT).max() <= 1.0


def test_row_permutation_equivariance():
    k, v, q, f, W, H0 = _rand(seed=6)
    K = k.shape[-1]
    P = np.random.default_rng(1).permutation(K)
    y, HT = oracle.forward(k, v, q, f, W, H0)
    y2, HT2 = oracle.forward(k[..., P], v, q[..., P], f, W, H0[:, :, P, :])
    np.testing.assert_allclose(HT2, HT[:, :, P, :], rtol=0, atol=1e-13)
    np.testing.assert_allclose(y2, y, rtol=0, atol=1e-13)


def test_column_permutation_equivariance():
    # v -> P v, W -> Pᵀ W P, H0 -> H0 P   gives   H -> H P and y -> P y
    k, v, q, f, W, H0 = _rand(seed=7)
    V = v.shape[-1]
    P = np.random.default_rng(2).permutation(V)
    y, HT = oracle.forward(k, v, q, f, W, H0)
    W2 = W[:, P][:, :, P]
    y2, HT2 = oracle.forward(k, v[..., P], q, f, W2, H0[..., P])
    np.testing.assert_allclose(HT2, HT[..., P], rtol=0, atol=1e-13)
    np.testing.assert_allclose(y2, y[..., P], rtol=0, atol=1e-13)


def test_batch_and_head_independence():
    k, v, q, f, W, H0 = _rand(B=3, H=2, seed=8)
    y, HT = oracle.forward(k, v, q, f, W, H0)
    k2, v2, q2, f2 = k.copy(), v.copy(), q.copy(), f.copy()
    k2[0] += 1.0; v2[2] *= -1; q2[0] = 0; f2[2] = 0.5
    y2, HT2 = oracle.forward(k2, v2, q2, f2, W, H0)
    np.testing.assert_array_equal(y2[1], y[1])
    np.testing.assert_array_equal(HT2[1], HT[1])
    # a single head on its own gives the same result
    y3, HT3 = oracle.forward(k[:, 1:], v[:, 1:], q[:, 1:], f[:, 1:], W[1:], H0[:, 1:])
    np.testing.assert_array_equal(y3, y[:, 1:])
    np.testing.assert_array_equal(HT3, HT[:, 1:])


def test_thread_count_does_not_change_results():
    k, v, q, f, W, H0 = _rand(B=3, H=3, T=6, seed=10)
    dy = np.random.default_rng(3).standard_normal(k.shape[:3] + (v.shape[-1],))
    g1 = oracle.backward(k, v, q, f, W, H0, dy, nthreads=1)
    g5 = oracle.backward(k, v, q, f, W, H0, dy, nthreads=5)
    for n in g1:
        np.testing.assert_array_equal(g1[n], g5[n])


def test_two_by_two_written_out():
    """K = V = 2, two steps, every scalar written out by hand (no matrix code)."""
    import math
    W = [[0.3, -0.7], [0.5, 0.2]]
    H = [[0.1, -0.2], [0.4, 0.05]]
    ks = [[1.0, -0.5], [0.25, 2.0]]
    vs = [[0.6, -0.3], [-1.2, 0.8]]
    qs = [[0.9, -1.1], [0.3, 0.7]]
    fs = [0.25, 0.8]
    ys = []
    for t in range(2):
        k1, k2 = ks[t]; v1, v2 = vs[t]; q1, q2 = qs[t]; ft = fs[t]
        a11 = H[0][0] * W[0][0] + H[0][1] * W[1][0] + k1 * v1
        a12 = H[0][0] * W[0][1] + H[0][1] * W[1][1] + k1 * v2
        a21 = H[1][0] * W[0][0] + H[1][1] * W[1][0] + k2 * v1
        a22 = H[1][0] * W[0][1] + H[1][1] * W[1][1] + k2 * v2
        H = [[ft * H[0][0] + (1 - ft) * math.tanh(a11), ft * H[0][1] + (1 - ft) * math.tanh(a12)],
             [ft * H[1][0] + (1 - ft) * math.tanh(a21), ft * H[1][1] + (1 - ft) * math.tanh(a22)]]
        ys.append([H[0][0] * q1 + H[1][0] * q2, H[0][1] * q1 + H[1][1] * q2])
    y, HT = oracle.forward(np.array(ks)[None, None], np.array(vs)[None, None], np.array(qs)[None, None],
                           np.array(fs)[None, None], np.array(W)[None],
                           np.array([[0.1, -0.2], [0.4, 0.05]])[None, None])
    np.testing.assert_allclose(y[0, 0], np.array(ys), rtol=0, atol=1e-15)
    np.testing.assert_allclose(HT[0, 0], np.array(H), rtol=0, atol=1e-15)


def _loss(k, v, q, f, W, H0, dy, dHT):
    y, HT = oracle.forward(k, v, q, f, W, H0, nthreads=1)
    return float((y * dy).sum() + (HT * dHT).sum())


@pytest.mark.parametrize("K,V", [(2, 2), (3, 4), (4, 2)])
def test_backward_finite_differences(K, V):
    k, v, q, f, W, H0 = _rand(B=2, H=2, T=6, K=K, V=V, seed=11 + K * V)
    r = np.random.default_rng(12)
    dy = r.standard_normal((2, 2, 6, V))
    dHT = r.standard_normal((2, 2, K, V))
    g = oracle.backward(k, v, q, f, W, H0, dy, dHT, nthreads=1)
    args = {"k": k, "v": v, "q": q, "f": f, "W": W, "H0": H0}
    names = {"k": "dk", "v": "dv", "q": "dq", "f": "df", "W": "dW", "H0": "dH0"}
    eps = 1e-6
    for name, arr in args.items():
        flat = arr.reshape(-1)
        idx = r.choice(flat.size, size=min(flat.size, 12), replace=False)
        for e in idx:
            old = flat[e]
            flat[e] = old + eps
            lp = _loss(dy=dy, dHT=dHT, **args)
            flat[e] = old - eps
            lm = _loss(dy=dy, dHT=dHT, **args)
            flat[e] = old
            fd = (lp - lm) / (2 * eps)
            an = g[names[name]].reshape(-1)[e]
            assert abs(fd - an) <= 1e-7 * max(1.0, abs(fd)), (name, e, fd, an)


def test_backward_closed_form_f1():
    # f = 1: H_t = H0, Z_t = tanh(H0 W + k_t v_tᵀ), dA = 0 (dZ = (1-f)G = 0):
    #   dH0 = dHT + sum_t q_t dy_tᵀ, dW = 0, dk = dv = 0, dq_t = H0 dy_t,
    #   df_t = <G_t, H0 - Z_t> with G_t = dHT + sum_{s>=t} q_s dy_sᵀ
    k, v, q, f, W, H0 = _rand(B=2, H=2, T=5, seed=13)
    f[:] = 1.0
    r = np.random.default_rng(14)
    dy = r.standard_normal(k.shape[:3] + (v.shape[-1],))
    dHT = r.standard_normal(H0.shape)
    g = oracle.backward(k, v, q, f, W, H0, dy, dHT)
    qdy = np.einsum("bhti,bhtj->bhtij", q, dy)
    np.testing.assert_allclose(g["dH0"], dHT + qdy.sum(2), rtol=0, atol=1e-13)
    assert np.all(g["dW"] == 0) and np.all(g["dk"] == 0) and np.all(g["dv"] == 0)
    np.testing.assert_allclose(g["dq"], np.einsum("bhij,bhtj->bhti", H0, dy), rtol=0, atol=1e-13)
    T = k.shape[2]
    for t in range(T):
        Gt = dHT + qdy[:, :, t:].sum(2)
        Zt = np.tanh(np.einsum("bhil,hlj->bhij", H0, W) + np.einsum("bhi,bhj->bhij", k[:, :, t], v[:, :, t]))
        np.testing.assert_allclose(g["df"][:, :, t], (Gt * (H0 - Zt)).sum((-1, -2)), rtol=0, atol=1e-12)


def test_backward_closed_form_W0_f0():
    # W = 0, f = 0: G_t = q_t dy_tᵀ (+ dHT at the last step), dA_t = G_t ⊙ (1 - Z_t²),
    # Z_t = H_t = tanh(k_t v_tᵀ); dk = dA v, dv = dAᵀ k, dq_t = H_t dy_t,
    # df_t = <G_t, H_{t-1} - Z_t>, dW = sum_t H_{t-1}ᵀ dA_t, dH0 = 0 (f = 0, W = 0)
    k, v, q, f, W, H0 = _rand(B=2, H=2, T=5, seed=15)
    W[:] = 0.0
    f[:] = 0.0
    r = np.random.default_rng(16)
    dy = r.standard_normal(k.shape[:3] + (v.shape[-1],))
    dHT = r.standard_normal(H0.shape)
    g = oracle.backward(k, v, q, f, W, H0, dy, dHT)
    Z = np.tanh(np.einsum("bhti,bhtj->bhtij", k, v))
    G = np.einsum("bhti,bhtj->bhtij", q, dy)
    G[:, :, -1] += dHT
    dA = G * (1 - Z ** 2)
    Hprev = np.concatenate([H0[:, :, None], Z[:, :, :-1]], axis=2)
    np.testing.assert_allclose(g["dk"], np.einsum("bhtij,bhtj->bhti", dA, v), rtol=0, atol=1e-13)
    np.testing.assert_allclose(g["dv"], np.einsum("bhtij,bhti->bhtj", dA, k), rtol=0, atol=1e-13)
    np.testing.assert_allclose(g["dq"], np.einsum("bhtij,bhtj->bhti", Z, dy), rtol=0, atol=1e-13)
    np.testing.assert_allclose(g["df"], (G * (Hprev - Z)).sum((-1, -2)), rtol=0, atol=1e-12)
    np.testing.assert_allclose(g["dW"], np.einsum("bhtil,bhtij->hlj", Hprev, dA), rtol=0, atol=1e-12)
    np.testing.assert_array_equal(g["dH0"], np.zeros_like(H0))


# ---------------------------------------------------------------- grouped q / k
# Grouped-value form (gist.science technical summary §2.2, tensor parallelism):
# k and q carry G groups of heads, head h uses group h // (H / G).

def _grouped(B=2, H=4, G=2, T=5, K=3, V=2, seed=21):
    k, v, q, f, W, H0 = _rand(B=B, H=H, T=T, K=K, V=V, seed=seed)
    r = np.random.default_rng(seed + 1)
    kg = r.standard_normal((B, G, T, K)) * 0.7
    qg = r.standard_normal((B, G, T, K)) * 0.7
    return kg, v, qg, f, W, H0


def test_grouped_heads_read_their_own_group():
    # Changing the k (or q) of group g changes exactly the heads g·H/G .. (g+1)·H/G - 1,
    # which pins the head -> group map (consecutive heads share, not h mod G).
    k, v, q, f, W, H0 = _grouped(H=6, G=3)
    y0, HT0 = oracle.forward(k, v, q, f, W, H0)
    for name in ("k", "q"):
        for g in range(3):
            k2, q2 = k.copy(), q.copy()
            (k2 if name == "k" else q2)[:, g] += 0.3
            y1, HT1 = oracle.forward(k2, v, q2, f, W, H0)
            changed = [h for h in range(6) if not np.array_equal(y1[:, h], y0[:, h])]
            assert changed == [2 * g, 2 * g + 1], (name, g, changed)
            if name == "q":   # q only enters the readout
                np.testing.assert_array_equal(HT1, HT0)


def test_one_group_with_equal_heads_gives_equal_heads():
    # G = 1 and every head given the same v, f, W, H0: all heads see the same
    # recurrence, so their outputs are bitwise equal; dk, dq are then H times
    # the gradient of one head with its own (ungrouped) k and q.
    k, v, q, f, W, H0 = _grouped(H=3, G=1)
    v[:] = v[:, :1]; f[:] = f[:, :1]; W[:] = W[:1]; H0[:] = H0[:, :1]
    y, HT = oracle.forward(k, v, q, f, W, H0)
    for h in range(1, 3):
        np.testing.assert_array_equal(y[:, h], y[:, 0])
        np.testing.assert_array_equal(HT[:, h], HT[:, 0])
    r = np.random.default_rng(22)
    dy1 = r.standard_normal(v[:, :1].shape)
    dy = np.repeat(dy1, 3, axis=1)
    g = oracle.backward(k, v, q, f, W, H0, dy)
    g1 = oracle.backward(k, v[:, :1], q, f[:, :1], W[:1], H0[:, :1], dy1)
    np.testing.assert_allclose(g["dk"], 3 * g1["dk"], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(g["dq"], 3 * g1["dq"], rtol=1e-13, atol=1e-15)


def test_grouped_backward_finite_differences():
    k, v, q, f, W, H0 = _grouped(H=4, G=2)
    r = np.random.default_rng(23)
    dy = r.standard_normal(v.shape)
    dHT = r.standard_normal(H0.shape)
    g = oracle.backward(k, v, q, f, W, H0, dy, dHT, nthreads=1)
    assert g["dk"].shape == k.shape and g["dq"].shape == q.shape
    args = {"k": k, "v": v, "q": q, "f": f, "W": W, "H0": H0}
    names = {"k": "dk", "v": "dv", "q": "dq", "f": "df", "W": "dW", "H0": "dH0"}
    eps = 1e-6
    for name, arr in args.items():
        flat = arr.reshape(-1)
        idx = r.choice(flat.size, size=min(flat.size, 10), replace=False)
        for e in idx:
            old = flat[e]
            flat[e] = old + eps
            lp = _loss(dy=dy, dHT=dHT, **args)
            flat[e] = old - eps
            lm = _loss(dy=dy, dHT=dHT, **args)
            flat[e] = old
            fd = (lp - lm) / (2 * eps)
            an = g[names[name]].reshape(-1)[e]
            assert abs(fd - an) <= 1e-7 * max(1.0, abs(fd)), (name, e, fd, an)


# ---------------------------------------------------------------- gate logits
# f_t = 1 / (1 + exp(-a_t)) from a gate logit a_t (reading of the forget gate's
# parameterisation ψ, gist.science technical summary §2.1).

def test_gate_logit_values():
    a = np.array([0.0, np.log(3.0), -np.log(3.0), 50.0, -800.0])
    np.testing.assert_allclose(oracle.gate_from_logit(a), [0.5, 0.75, 0.25, 1.0, 0.0], rtol=1e-15, atol=1e-300)


def test_gate_logit_forward_is_the_forward_of_the_gate_value():
    # a = log(f / (1 - f)) inverts the logistic: the logit path must reproduce
    # the value path (a flipped sign would give the gate 1 - f instead)
    k, v, q, f, W, H0 = _rand(seed=31)
    a = np.log(f / (1.0 - f))
    y, HT = oracle.forward(k, v, q, f, W, H0)
    ya, HTa = oracle.forward(k, v, q, a, W, H0, f_is_logit=True)
    np.testing.assert_allclose(ya, y, rtol=0, atol=1e-13)
    np.testing.assert_allclose(HTa, HT, rtol=0, atol=1e-13)
    # a saturated logit is f = 1 exactly: the state stays H0
    _, HT1 = oracle.forward(k, v, q, np.full_like(f, 50.0), W, H0, f_is_logit=True)
    np.testing.assert_array_equal(HT1, H0)


def test_gate_logit_backward_finite_differences():
    k, v, q, f, W, H0 = _rand(B=2, H=2, T=6, K=3, V=4, seed=33)
    a = np.random.default_rng(34).standard_normal(f.shape) * 2.0
    r = np.random.default_rng(35)
    dy = r.standard_normal(v.shape)
    dHT = r.standard_normal(H0.shape)
    g = oracle.backward(k, v, q, a, W, H0, dy, dHT, nthreads=1, f_is_logit=True)
    eps = 1e-6
    flat = a.reshape(-1)
    for e in range(flat.size):
        old = flat[e]
        flat[e] = old + eps
        yp, HTp = oracle.forward(k, v, q, a, W, H0, nthreads=1, f_is_logit=True)
        flat[e] = old - eps
        ym, HTm = oracle.forward(k, v, q, a, W, H0, nthreads=1, f_is_logit=True)
        flat[e] = old
        fd = (((yp - ym) * dy).sum() + ((HTp - HTm) * dHT).sum()) / (2 * eps)
        an = g["df"].reshape(-1)[e]
        assert abs(fd - an) <= 1e-7 * max(1.0, abs(fd)), (e, fd, an)
    # the other gradients do not depend on how f was given
    gv = oracle.backward(k, v, q, oracle.gate_from_logit(a), W, H0, dy, dHT, nthreads=1)
    for n in ("dk", "dv", "dq", "dW", "dH0"):
        np.testing.assert_array_equal(g[n], gv[n])

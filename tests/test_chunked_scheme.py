"""The chunked form's bf16-part arithmetic, modelled in numpy (CPU only).

GDN_FLAG_CHUNKED runs a chain in chunks of T = 64 tokens with the delta
rule's chunked "WY" form (the Gated Delta Networks paper by Yang, Kautz and
Hatamizadeh derives it): per chunk X^T | Y^T = S [K; Q]^T, U^T = (V^T -
X^T diag(Gamma)) Ab^T with Ab = (I + L)^-1 diag(beta), O^T = scale (Y^T
diag(Gamma) + U^T M^T), S <- Gamma_{T-1} S + (U^T diag(r)) K.  The kernel
forms every product on the tensor cores from bf16 parts of its operands
(x = x1 + x2 (+ x3), x2 = bf16(x - x1), ...), with f32 accumulation.

This model keeps that part structure (which operands are split into how
many parts, which part products are formed) and rounds each part product to
f32 once; it is not bit-exact to the tensor cores' accumulation order and
shares no code with the CUDA path.  Against the exact recurrence (token by
token, float64) it pins the choice of parts: the kernel's choice stays
within a few times the f32 token walk's own rounding error, and dropping a
part from any of the three products that feed the state is detected."""
import numpy as np
import pytest
import torch

T = 64
D_K, D_V = 128, 8
N = 1024
SCALE = D_K ** -0.5

# part products (i, j) of U^T = P^T Ab^T, by part index of P and of Ab
P_AB_KERNEL = [(0, 0), (0, 1), (1, 0), (0, 2), (1, 1), (2, 0)]   # weight down to 2^-16
KERNEL = dict(s_parts=2, ur_parts=3, p_ab=P_AB_KERNEL)


def _bf16(x):
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


def _parts(x, n):
    """x = x1 + ... + xn, each a bf16 value, x_{i+1} = bf16(x - x1 - ... - xi)."""
    rest, out = x.astype(np.float32), []
    for _ in range(n):
        p = _bf16(rest)
        out.append(p)
        rest = (rest - p).astype(np.float32)
    return out


def _prod(a, b):
    # a product of bf16 parts, exact, rounded to f32 once
    return (a.astype(np.float64) @ b.astype(np.float64)).astype(np.float32)


def _problem(a_lo, seed):
    """A chain shaped like the long-chain workload: unit-norm bf16 k and q,
    bf16 v, a = exp(g) uniform in [a_lo, 1], beta = sigmoid(N(0,1))."""
    rng = np.random.default_rng(seed)
    k = rng.standard_normal((N, D_K))
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    q = rng.standard_normal((N, D_K))
    q /= np.linalg.norm(q, axis=1, keepdims=True)
    v = rng.standard_normal((N, D_V))
    g = np.log(rng.uniform(a_lo, 1.0, N)).astype(np.float32)
    beta = (1.0 / (1.0 + np.exp(-rng.standard_normal(N)))).astype(np.float32)
    s0 = (0.1 * rng.standard_normal((D_V, D_K))).astype(np.float32)
    return _bf16(k), _bf16(q), _bf16(v), g, beta, s0


def _exact(k, q, v, g, beta, s0):
    S, O = s0.astype(np.float64), np.zeros((N, D_V))
    for t in range(N):
        Sp = np.exp(np.float64(g[t])) * S
        S = Sp + np.float64(beta[t]) * np.outer(v[t] - Sp @ k[t], k[t])
        O[t] = SCALE * S @ q[t]
    return S, O


def _walk_f32(k, q, v, g, beta, s0):
    S, O = s0.copy(), np.zeros((N, D_V), np.float32)
    for t in range(N):
        Sp = np.float32(np.exp(g[t])) * S
        S = (Sp + beta[t] * np.outer(v[t] - Sp @ k[t], k[t])).astype(np.float32)
        O[t] = SCALE * S @ q[t]
    return S, O


def _chunked(k, q, v, g, beta, s0, s_parts, ur_parts, p_ab):
    S, O = s0.copy(), np.zeros((N, D_V), np.float32)
    below = np.arange(T)[None, :] < np.arange(T)[:, None]
    on_or_below = np.arange(T)[None, :] <= np.arange(T)[:, None]
    for c0 in range(0, N, T):
        K, Q, V, b = k[c0:c0 + T], q[c0:c0 + T], v[c0:c0 + T], beta[c0:c0 + T]
        a = np.exp(g[c0:c0 + T]).astype(np.float32)
        # R[t][i] = a_{i+1} ... a_t, Gamma_t = a_0 ... a_t
        R, Gam = np.zeros((T, T), np.float32), np.zeros(T, np.float32)
        for t in range(T):
            run = np.float32(1.0)
            for i in range(t, -1, -1):
                R[t, i] = run
                run = np.float32(run * a[i])
            Gam[t] = run
        r = R[T - 1]
        L = np.where(below, b[:, None] * (_prod(K, K.T) * R), 0.0).astype(np.float32)
        M = np.where(on_or_below, _prod(Q, K.T) * R, 0.0).astype(np.float32)
        Ab = (np.linalg.inv(np.eye(T) + L.astype(np.float64)) * b[None, :]).astype(np.float32)
        s = _parts(S, s_parts)
        XT = sum(_prod(p, K.T) for p in s)
        YT = sum(_prod(p, Q.T) for p in s)
        PT = (V.T - Gam[None, :] * XT).astype(np.float32)
        pp, ap = _parts(PT, 3), _parts(Ab, 3)
        UT = sum(_prod(pp[i], ap[j].T) for i, j in p_ab)
        up, mp = _parts(UT, 2), _parts(M, 2)
        UM = sum(_prod(up[i], mp[j].T) for i, j in [(0, 0), (0, 1), (1, 0)])
        O[c0:c0 + T] = (SCALE * (Gam[None, :] * YT + UM)).T
        ur = _parts(UT * r[None, :], ur_parts)
        S = (Gam[T - 1] * S + sum(_prod(p, K) for p in ur)).astype(np.float32)
    return S, O


def _rel(x, ref):
    return float(np.linalg.norm(x - ref) / np.linalg.norm(ref))


# a uniform in [0.5, 1] (the long-chain workload's gate) and in [0.995, 1]
# (slow decay: rounding persists longest)
CASES = [(0.5, 5), (0.995, 5)]
STATE_FACTOR = 8.0     # times the f32 walk's own state error
STATE_FLOOR = 2e-7
OUT_BOUND = 4e-6


def _errors(case, **scheme):
    prob = _problem(*case)
    S, O = _exact(*prob)
    Sc, Oc = _chunked(*prob, **scheme)
    return _rel(Sc, S), float(np.abs(Oc - O).max())


@pytest.mark.parametrize("case", CASES)
def test_kernel_parts_stay_near_f32_walk(case):
    prob = _problem(*case)
    S, O = _exact(*prob)
    Sw, _ = _walk_f32(*prob)
    walk = _rel(Sw, S)
    st, out = _errors(case, **KERNEL)
    assert st <= max(STATE_FACTOR * walk, STATE_FLOOR), (st, walk)
    assert out <= OUT_BOUND, out
    # and far inside the parity tolerances (1e-3 relative Frobenius on f32
    # states, 2e-3 max-abs on outputs)
    assert st < 1e-5 and out < 1e-5


@pytest.mark.parametrize("drop", ["state", "update", "p_ab"])
def test_dropping_a_part_is_detected(drop):
    """Each of the three state-feeding products with one part fewer (S in 1
    part, U^T diag(r) in 1 part, U^T from the leading part product only)
    breaks one of the bounds above in at least one case."""
    scheme = dict(KERNEL)
    if drop == "state":
        scheme["s_parts"] = 1
    elif drop == "update":
        scheme["ur_parts"] = 1
    else:
        scheme["p_ab"] = [(0, 0)]
    broken = False
    for case in CASES:
        prob = _problem(*case)
        S, _ = _exact(*prob)
        Sw, _ = _walk_f32(*prob)
        st, out = _errors(case, **scheme)
        broken |= st > max(STATE_FACTOR * _rel(Sw, S), STATE_FLOOR) or out > OUT_BOUND
    assert broken

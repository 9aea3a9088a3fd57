"""Pins of the acceptance-step oracle (LoopSpec article: the final check tries the
first draft, then the fallback, and restarts only after both are rejected; greedy
decoding keeps the original model's token, sampling keeps its distribution).

Each test pins the oracle to something outside it: the distribution-preservation
theorem of speculative sampling (exact marginal and Monte Carlo), greedy
exactness, and closed forms for the special cases."""
import numpy as np
import pytest

from oracle import accept as AC


def _logits(rng, V, spread=2.0):
    return rng.standard_normal(V) * spread


def _near(z, rng, eps):
    return z + eps * rng.standard_normal(len(z))


@pytest.mark.parametrize("temperature", [1.0, 0.7])
@pytest.mark.parametrize("with_fallback", [False, True])
def test_emitted_token_is_distributed_as_the_final_distribution(temperature, with_fallback):
    rng = np.random.default_rng(10)
    for _ in range(20):
        zp = _logits(rng, 40)
        zq = _near(zp, rng, 1.5)          # early loops: a blurred version of the final logits
        zf = _near(zp, rng, 0.5) if with_fallback else None   # deeper: closer to the final ones
        out = AC.output_distribution(zp, zq, zf, temperature)
        np.testing.assert_allclose(out, AC.softmax(zp, temperature), rtol=0, atol=1e-12)


def test_monte_carlo_of_the_procedure_matches_the_final_distribution():
    """The step-by-step procedure (draws by inverse CDF from uniforms), sampled
    200 000 times on a 6-token vocabulary, emits each token with frequency p(v)."""
    rng = np.random.default_rng(11)
    zp = np.array([1.2, 0.1, -0.5, 0.9, -1.5, 0.3])
    zq = np.array([0.2, 1.1, -0.2, 0.1, -0.3, 0.4])
    zf = np.array([1.0, 0.6, -0.6, 0.5, -1.0, 0.2])
    p = AC.softmax(zp, 1.0)
    q1 = AC.softmax(zq, 1.0)
    n = 200_000
    u = rng.random((n, 5))
    counts = np.zeros(6)
    for i in range(n):
        x1 = AC.draw(q1, u[i, 0])
        x2 = AC.fallback_token(zq, zf, x1, 1.0, u[i, 1])
        ok, tok, path = AC.accept_position(zp, zq, zf, x1, x2, u[i, 2:5], 1.0)
        counts[x1 if ok else tok] += 1
    freq = counts / n
    sigma = np.sqrt(p * (1 - p) / n)
    assert np.all(np.abs(freq - p) < 5 * sigma), (freq, p)


def test_greedy_keeps_the_original_models_token():
    rng = np.random.default_rng(12)
    V, k = 50, 6
    for _ in range(200):
        zp = rng.standard_normal((k, V))
        zq = zp + rng.standard_normal((k, V)) * 0.8
        zf = zp + rng.standard_normal((k, V)) * 0.3
        x1 = np.argmax(zq, axis=1)
        x2 = np.array([AC.fallback_token(zq[j], zf[j], int(x1[j]), 0, 0.0) for j in range(k)])
        n, tok, path = AC.accept_block(zp, zq, zf, x1, x2, np.zeros((k, 3)), 0)
        best = np.argmax(zp, axis=1)
        assert np.array_equal(x1[:n], best[:n])           # accepted drafts are the model's tokens
        if n < k:
            assert x1[n] != best[n] and tok == best[n]      # the emitted token is the model's
            assert path == (AC.FALLBACK if x2[n] == best[n] and AC.fallback_gate(zq[n], zf[n], int(x1[n]))
                            else AC.RESTART)


def test_closed_forms():
    rng = np.random.default_rng(13)
    zp = _logits(rng, 30)
    # draft equal to the final distribution: every proposal is accepted
    for x1 in range(30):
        assert AC.accept_position(zp, zp, None, x1, 0, (0.999999, 0.0, 0.0), 1.0)[0]
    # the fallback never raises the restart probability: Z1 (1 - sum min(p1, q2)) <= Z1
    for _ in range(20):
        zp = _logits(rng, 30)
        zq = _near(zp, rng, 1.5)
        zf = _near(zp, rng, 0.4)
        p, q1 = AC.softmax(zp, 1.0), AC.softmax(zq, 1.0)
        z1 = np.maximum(p - q1, 0).sum()
        p1 = AC.residual(p, q1)
        q2 = AC.fallback_distribution(zq, zf, 1.0)
        assert z1 * (1 - np.minimum(p1, q2).sum()) <= z1 + 1e-15
    # inverse-CDF draw: u = 0 gives the first token with mass, u -> 1 the last
    w = np.array([0.0, 0.2, 0.0, 0.5, 0.3])
    assert AC.draw(w, 0.0) == 1 and AC.draw(w, 0.999) == 4 and AC.draw(w, 0.25) == 3

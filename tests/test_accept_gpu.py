"""The acceptance kernel (ripe_accept) against the acceptance oracle, through the
C ABI: greedy and sampling temperatures, with and without a fallback.  The
uniforms are drawn so that no decision sits within 1e-4 (relative) of its
threshold, where fp32 and fp64 could round to different sides; every decision is
then unique and compared exactly."""
import numpy as np
import pytest
import torch

from oracle import accept as AC

pytestmark = pytest.mark.gpu

MARGIN = 1e-4


def _robust(zp, zq, zf, x1, temperature, rng):
    """Uniforms (u0, u1, u2) and a fallback token whose decisions are clear of their
    thresholds, and whose gate is not a near-tie."""
    p, q1 = AC.softmax(zp, temperature), AC.softmax(zq, temperature)
    if zf is not None:
        g1, g2 = AC.softmax(zf, 1.0)[x1], AC.softmax(zq, 1.0)[x1]
        if abs(g1 - g2) <= MARGIN * max(g1, g2):
            return None
    for _ in range(100):
        u = rng.random(3)
        x2 = AC.fallback_token(zq, zf, x1, temperature, rng.random()) if zf is not None else 0
        if temperature == 0:
            return u, x2
        if abs(u[0] * q1[x1] - p[x1]) <= MARGIN * max(p[x1], q1[x1]):
            continue
        p1 = AC.residual(p, q1)
        if p1.sum() == 0:
            p1 = p
        w = p1
        if zf is not None and AC.fallback_gate(zq, zf, x1):
            q2 = AC.fallback_distribution(zq, zf, temperature)
            if q2.sum() > 0:
                if abs(u[1] * q2[x2] - p1[x2]) <= MARGIN * max(p1[x2], q2[x2]):
                    continue
                r2 = AC.residual(p1, q2)
                w = r2 if r2.sum() > 0 else p1
        c = np.cumsum(w) / w.sum()
        if np.min(np.abs(c - u[2])) <= MARGIN:
            continue
        return u, x2
    return None


@pytest.mark.parametrize("temperature", [0.0, 0.8, 1.0])
@pytest.mark.parametrize("with_fallback", [False, True])
@pytest.mark.parametrize("V", [333, 32000])
def test_accept_matches_oracle(temperature, with_fallback, V):
    from depth_planed_kv_b200.ripe import ripe_accept
    rng = np.random.default_rng(int(temperature * 10) + 100 * with_fallback + V)
    nseq, k = 24, 5
    zp = rng.standard_normal((nseq, k, V)).astype(np.float32) * 3
    zq = (zp + rng.standard_normal((nseq, k, V)).astype(np.float32) * 1.2).astype(np.float32)
    zf = (zp + rng.standard_normal((nseq, k, V)).astype(np.float32) * 0.5).astype(np.float32) if with_fallback else None
    x1 = np.zeros((nseq, k), np.int32)
    x2 = np.zeros((nseq, k), np.int32)
    u = np.zeros((nseq, k, 3), np.float32)
    for b in range(nseq):
        for j in range(k):
            while True:
                q1 = AC.softmax(zq[b, j], temperature)
                x = AC.draw(q1, rng.random()) if temperature > 0 else int(np.argmax(zq[b, j]))
                # a quarter of the drafts are the final argmax, so blocks run past position 0
                if rng.random() < 0.25:
                    x = int(np.argmax(zp[b, j]))
                got = _robust(zp[b, j].astype(np.float64), zq[b, j].astype(np.float64),
                              None if zf is None else zf[b, j].astype(np.float64), x, temperature, rng)
                if got is not None:
                    break
            x1[b, j] = x
            u[b, j], x2[b, j] = got[0], got[1]
    dev = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a)).cuda()
    n_acc, tok, path = ripe_accept(dev(zp), dev(zq), dev(zf), dev(x1), dev(x2) if with_fallback else None,
                                   dev(u), temperature)
    torch.cuda.synchronize()
    n_acc, tok, path = n_acc.cpu().numpy(), tok.cpu().numpy(), path.cpu().numpy()
    for b in range(nseq):
        ref = AC.accept_block(zp[b].astype(np.float64), zq[b].astype(np.float64),
                              None if zf is None else zf[b].astype(np.float64), x1[b], x2[b],
                              u[b].astype(np.float64), temperature)
        assert (int(n_acc[b]), int(tok[b]), int(path[b])) == ref, (b, (n_acc[b], tok[b], path[b]), ref)
    if temperature == 0:   # greedy: the emitted token is always the final argmax
        for b in range(nseq):
            if n_acc[b] < k:
                assert tok[b] == np.argmax(zp[b, n_acc[b]])

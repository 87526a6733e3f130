"""Test helpers: expert banks built by the oracle's quantizer from seeded
synthetic weights, device upload helpers, and the tolerance check."""
import numpy as np

from streamed_quantized_expert_b200 import synth

_CACHE = {}


def oracle_bank(orc, n_rows, H, I, g, b_gu, b_d, seed=0):
    """uint8 [n_rows, slot_bytes]: row r = quantized synth.expert_weights(seed, r)."""
    key = (n_rows, H, I, g, b_gu, b_d, seed)
    if key not in _CACHE:
        rows = [orc.build_slot(*synth.expert_weights(seed, r, H, I), g, b_gu, b_d) for r in range(n_rows)]
        _CACHE[key] = np.stack(rows)
    return _CACHE[key]


def assert_close(y, ref, tol=2e-2, what="y"):
    """|y - r| <= tol * max(|r|, rms of r's row), elementwise."""
    y = np.asarray(y, np.float64)
    ref = np.asarray(ref, np.float64)
    assert y.shape == ref.shape, (y.shape, ref.shape)
    rms = np.sqrt(np.mean(ref ** 2, axis=-1, keepdims=True))
    bound = tol * np.maximum(np.abs(ref), rms)
    err = np.abs(y - ref)
    bad = err > bound
    normwise = float(np.max(np.linalg.norm(y - ref, axis=-1) / np.maximum(np.linalg.norm(ref, axis=-1), 1e-30)))
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; max err/bound "
                           f"{float(np.max(err / np.maximum(bound, 1e-30))):.3g}; normwise {normwise:.3g}")
    return normwise


def oracle_bank_parallel(orc, n_rows, H, I, g, b_gu, b_d, seed=0):
    """oracle_bank built on a thread pool (the oracle's C calls release the GIL)."""
    import os
    from concurrent.futures import ThreadPoolExecutor

    key = (n_rows, H, I, g, b_gu, b_d, seed)
    if key not in _CACHE:
        with ThreadPoolExecutor(max_workers=os.cpu_count() or 1) as ex:
            rows = list(ex.map(lambda r: orc.build_slot(*synth.expert_weights(seed, r, H, I), g, b_gu, b_d),
                               range(n_rows)))
        _CACHE[key] = np.stack(rows)
    return _CACHE[key]


def oracle_rows_parallel(orc, x, geom, ids, w, slots, tokens=None, chunk=256):
    """The oracle's y rows for `tokens` (default: every token), evaluated pair
    by pair on a thread pool.  Each (token, rank) pair is the oracle's FFN of
    that one token with k = 1 and weight 1, which is exactly o_{t,j}; pairs are
    grouped by slot (each group dequantises its slot once) and y_t is then
    summed over j in rank order as the oracle sums it, so the rows equal the
    single-call oracle's bit for bit."""
    import os
    from concurrent.futures import ThreadPoolExecutor

    H = geom[0]
    T, k = ids.shape
    tok = np.arange(T) if tokens is None else np.asarray(tokens)
    o = np.zeros((tok.size, k, H), np.float64)
    groups = {}
    for ti, t in enumerate(tok):
        for j in range(k):
            groups.setdefault(slots[int(ids[t, j])].ctypes.data, []).append((ti, j, int(t), int(ids[t, j])))
    jobs = []
    for lst in groups.values():
        for c0 in range(0, len(lst), chunk):
            jobs.append(lst[c0:c0 + chunk])

    def run(job):
        xs = np.stack([x[t] for _, _, t, _ in job])
        one = orc.expert_ffn(xs, *geom, np.zeros((len(job), 1), np.int32), np.ones((len(job), 1)),
                             [slots[job[0][3]]])
        for (ti, j, _, _), row in zip(job, one):
            o[ti, j] = row

    with ThreadPoolExecutor(max_workers=os.cpu_count() or 1) as ex:
        list(ex.map(run, jobs))
    y = np.zeros((tok.size, H), np.float64)
    wf = np.asarray(w, np.float64)
    for j in range(k):
        y += wf[tok, j][:, None] * o[:, j]
    return y

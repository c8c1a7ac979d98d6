"""Mutation check of the oracle's pins (run by hand; not collected by pytest).

    python tests/mutation_check.py

Plants one plausible mistake at a time in a copy of oracle/ (a dropped
rescale, a wrong sign, a wrong index or block size, exp for exp2, an
off-by-one in the fixed summation order, ...: in the contract's tile loop, in
the plain reading of the softmax, in the quantizers and in the numerics) and
runs the CPU pins of the oracle on the copy.  Every mistake must make at least
one pin fail; the script prints CAUGHT or MISSED for each and a total.
"""
import os
import shutil
import subprocess
import sys
import tempfile

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
M = [
 ("sage_oracle.py", "l = rn(rn(l * alpha) + rn(y.sum(axis=1)))", "l = rn(l + rn(y.sum(axis=1)))"),
 ("sage_oracle.py", "acc = rn(rn(acc * alpha[:, None]) + rn(p8 @ Vt[:, j0:j1].T))\n        m = m_new\n    o = np.asarray(fma(", "acc = rn(rn(acc) + rn(p8 @ Vt[:, j0:j1].T))\n        m = m_new\n    o = np.asarray(fma("),
 ("sage_oracle.py", "m_new = m if two_pass else np.maximum(m, tmax)", "m_new = m if two_pass else tmax"),
 ("sage_oracle.py", "e_off = np.asarray(fma(np.float64(-s_bias), c_full, e[:, None])", "e_off = np.asarray(fma(np.float64(s_bias), c_full, e[:, None])"),
 ("sage_oracle.py", "rn(1.0 / l)[:, None], out_add[None, :])", "rn(1.0 / l)[:, None], 0.0 * out_add[None, :])"),
 ("sage_oracle.py", "f = rn32(x.astype(np.float64) - nf.astype(np.float64))", "f = rn32(nf.astype(np.float64) - x.astype(np.float64))"),
 ("sage_oracle.py", "bits = p.view(np.uint32) + (xr.view(np.uint32) << np.uint32(23))", "bits = p.view(np.uint32) + (xr.view(np.uint32) << np.uint32(22))"),
 ("sage_oracle.py", "EXP2_C = tuple(np.float32(v) for v in (1.0, 0.7029417753219604,", "EXP2_C = tuple(np.float32(v) for v in (1.0, 0.6931471805599453,"),
 ("sage_oracle.py", "l = rn(rn(l * alpha) + rn(p.sum(axis=1)))", "l = rn(l + rn(p.sum(axis=1)))"),
 ("sage_oracle.py", "acc = rn(rn(acc * alpha[:, None]) + rn(p8 @ Vt[:, j0:j1].T))\n        m = m_new\n    o = rn(", "acc = rn(rn(acc) + rn(p8 @ Vt[:, j0:j1].T))\n        m = m_new\n    o = rn("),
 ("sage_oracle.py", "p8 = np.asarray(quant_p(rn(np.float64(E4M3_MAX) * p)), dtype=np.float64)", "p8 = np.asarray(quant_p(rn(np.float64(256.0) * p)), dtype=np.float64)"),
 ("sage_oracle.py", "o = rn(acc * out_mult[None, :] / (np.float64(E4M3_MAX) * l)[:, None] + out_add[None, :])", "o = rn(acc * out_mult[None, :] / l[:, None] + out_add[None, :])"),
 ("sage_oracle.py", "m_new = np.maximum(m, t.max(axis=1))", "m_new = t.max(axis=1)"),
 ("sage_oracle.py", "alpha = np.where(np.isneginf(m), 0.0, np.asarray(exp2(rn(m - m_new)), dtype=np.float64))\n        p = ", "alpha = np.where(np.isneginf(m), 0.0, np.asarray(exp2(rn(m_new - m)), dtype=np.float64))\n        p = "),
 ("sage_oracle.py", "return rn32(np.exp2(np.asarray(x, dtype=np.float64)))", "return rn32(np.exp(np.asarray(x, dtype=np.float64)))"),
 ("sage_oracle.py", "inv = np.where(nz, np.float32(INT8_MAX) / safe, np.float32(0)).astype(np.float32)\n    inv_tok", "inv = np.where(nz, np.float32(128.0) / safe, np.float32(0)).astype(np.float32)\n    inv_tok"),
 ("sage_oracle.py", "codes = np.clip(np.rint(prod), -INT8_MAX, INT8_MAX)", "codes = np.clip(np.trunc(prod), -INT8_MAX, INT8_MAX)"),
 ("sage_oracle.py", "kc = round_f32_to_bf16((k32 - mean32[:, None, :, :])", "kc = round_f32_to_bf16((k32 + mean32[:, None, :, :])"),
 ("sage_oracle.py", "(mean - vmin).astype(np.float32))", "(vmin - mean).astype(np.float32))"),
 ("sage_oracle.py", "for n in range(c * SUM_BLOCK, min(N, (c + 1) * SUM_BLOCK)):", "for n in range(c * SUM_BLOCK, min(N, (c + 1) * SUM_BLOCK) - 1):"),
 ("sage_oracle.py", "    o = SUM_LANES // 2\n", "    o = SUM_LANES // 4\n"),
 ("sage_oracle.py", "starts.extend(range(a, e, QK_BLOCK))", "starts.extend(range(a, e, 32))"),
 ("sage_oracle.py", "return f64_to_bf16_bits(s / np.float64(N)).reshape(B, H, D)", "return f64_to_bf16_bits(s / np.float64(N - 1)).reshape(B, H, D)"),
 ("sage_oracle.py", "return np.repeat(scale, QK_BLOCK, axis=-1)", "return np.repeat(scale, 128, axis=-1)[..., :Np]"),
 ("sage_oracle.py", "p_codes[:, j0:j1] = e4m3_encode(y.astype(np.float32))", "p_codes[:, j0:j1] = e4m3_encode((y * 0.5).astype(np.float32))"),
 ("sage_oracle.py", "sl2e = exp2_scale(sm_scale)\n    rows = np.arange(N) if rows is None else np.asarray(rows)\n    out = np.zeros((B, rows.shape[0], H, D), dtype=np.float32)\n    heads = [(b, h) for b in range(B) for h in range(H)] if heads is None else heads\n    for b, h in heads:\n        S = q_codes", "sl2e = np.float32(sm_scale)\n    rows = np.arange(N) if rows is None else np.asarray(rows)\n    out = np.zeros((B, rows.shape[0], H, D), dtype=np.float32)\n    heads = [(b, h) for b in range(B) for h in range(H)] if heads is None else heads\n    for b, h in heads:\n        S = q_codes"),
]
tests = ("tests/test_oracle_sage.py tests/test_oracle_numerics.py tests/test_oracle_plain.py "
         "tests/test_oracle_granularity.py tests/test_oracle_p_codes.py")
caught = 0
work = tempfile.mkdtemp(prefix='oracle_mutants_')
for i, (f, a, b) in enumerate(M):
    mut = os.path.join(work, str(i))
    for d in ('oracle', 'synth', 'tests'):
        shutil.copytree(os.path.join(ROOT, d), os.path.join(mut, d))
    p = os.path.join(mut, 'oracle', f)
    s = open(p).read()
    assert s.count(a) == 1, ('NOT UNIQUE', i, s.count(a), a[:70])
    open(p, 'w').write(s.replace(a, b, 1))
    r = subprocess.run(f'timeout 600 {sys.executable} -m pytest {tests} -q -x -p no:cacheprovider 2>&1 | tail -1', shell=True,
                       cwd=mut, capture_output=True, text=True)
    ok = 'failed' in r.stdout or 'error' in r.stdout
    caught += ok
    print(('CAUGHT ' if ok else 'MISSED ') + f"{i:2d} " + a.splitlines()[0][:70], '|', r.stdout.strip(), flush=True)
print(f"{caught} of {len(M)} caught")
shutil.rmtree(work, ignore_errors=True)
sys.exit(0 if caught == len(M) else 1)

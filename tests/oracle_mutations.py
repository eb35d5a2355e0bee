"""Mutation check of the CPU oracle's pins (run by hand; pytest does not collect it).

Each entry plants one plausible mistake (a dropped term, a wrong index or
bound, a flipped comparison or sign, another rounding) in a temporary copy of
``oracle/`` and runs the oracle's CPU pins (``tests/test_oracle_*.py``) on that
copy; the tracked files are never written. A mistake counts as caught
("KILLED") only when the pins ran and at least one failed (pytest exit 1); a
collection error or a timeout is reported as an error. A pin set is adequate
when every mistake is caught.

    python tests/oracle_mutations.py
"""
import os
import shutil
import subprocess
import sys
import tempfile

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PINS = ["tests/test_oracle_quant.py", "tests/test_oracle_route.py", "tests/test_oracle_attention.py",
        "tests/test_oracle_kv_cache.py"]

M = [
 ('oracle/quant.py', 's = np.float32(amax / np.float32(127.0))', 's = np.float32(amax / np.float32(128.0))'),
 ('oracle/quant.py', 'q = np.rint(ratio)', 'q = np.floor(ratio + 0.5)'),
 ('oracle/quant.py', 'out[i] = q8[r0:r1].astype(np.int64).sum(axis=0)', 'out[i] = q8[r0:max(r0, r1 - 1)].astype(np.int64).sum(axis=0)'),
 ('oracle/quant.py', 'mid = min(t1, t0 + 32)', 'mid = min(t1, t0 + 31)'),
 ('oracle/quant.py', 'out[j, 1] = k8[mid:t1]', 'out[j, 1] = k8[mid:max(mid, t1 - 1)]'),
 ('oracle/quant.py', 'out[t0:t1] = x8[t0:t1].astype(np.float64) * float(scale[b])', 'out[t0:t1] = x8[t0:t1].astype(np.float64) * float(scale[min(b + 1, len(scale) - 1)])'),
 ('oracle/quant.py', 'amax = np.float32(np.max(np.abs(blk)))', 'amax = np.float32(np.max(blk))'),
 ('oracle/route.py', 'return prod / n_j[None, :]', 'return prod / 64.0'),
 ('oracle/route.py', 'prod = dot.astype(np.float64) * k_scale.astype(np.float64)[None, :]', 'prod = dot.astype(np.float64) * 1.0'),
 ('oracle/route.py', 'PK = PK_half.sum(axis=1)', 'PK = PK_half[:, 0]'),
 ('oracle/route.py', 'var = _sequential_sum((R - mu[:, None]) ** 2) / nR', 'var = _sequential_sum((R - mu[:, None]) ** 2) / max(1, nR - 1)'),
 ('oracle/route.py', 'keep[i, routed] = R[i] >= T', 'keep[i, routed] = R[i] > T'),
 ('oracle/route.py', 'T = mu[i] + tau * sigma[i]', 'T = mu[i] - tau * sigma[i]'),
 ('oracle/route.py', 'routed = (K_ROWS * np.arange(nKB)) >= n_prefix\n    R = s[:, routed]\n    nR = R.shape[1]\n    keep = np.zeros((nQB, nKB), dtype=bool)\n    band', 'routed = (K_ROWS * np.arange(nKB)) > n_prefix\n    R = s[:, routed]\n    nR = R.shape[1]\n    keep = np.zeros((nQB, nKB), dtype=bool)\n    band'),
 ('oracle/route.py', 'or Q_ROWS * i < n_prefix\n', 'or Q_ROWS * i <= n_prefix\n'),
 ('oracle/route.py', 'or R[i].max() == R[i].min()', 'or False'),
 ('oracle/route.py', 'band[i, routed] = np.abs(R[i] - T) <= BAND_REL * sigma[i]', 'band[i, routed] = np.abs(R[i] - T) <= BAND_REL'),
 ('oracle/route.py', 'return n_routed - int(math.floor(sparsity * n_routed))', 'return n_routed - int(math.ceil(sparsity * n_routed))'),
 ('oracle/route.py', 'order = ridx[np.lexsort((ridx, -s[i, ridx]))]', 'order = ridx[np.lexsort((-ridx, -s[i, ridx]))]'),
 ('oracle/route.py', 'T = s[i, order[k - 1]]', 'T = s[i, order[min(k, len(order) - 1)]]'),
 ('oracle/route.py', '            keep[i, ~routed] = True\n            if k == 0:', '            if k == 0:'),
 ('oracle/route.py', 'if Q_ROWS * i < n_prefix or k >= nR:', 'if Q_ROWS * i < n_prefix or k > nR:'),
 ('oracle/route.py', 'mu = _sequential_sum(R) / nR\n        sigma = np.sqrt(_sequential_sum((R - mu[:, None]) ** 2) / nR)', 'mu = _sequential_sum(R) / nR\n        sigma = np.sqrt(_sequential_sum((R - mu[:, None]) ** 2) / max(1, nR - 1))'),
 ('oracle/attention.py', '        mid = min(t1, t0 + 32)\n        return', '        mid = min(t1, t0 + 31)\n        return'),
 ('oracle/attention.py', 'kbar = float(k_scale[j]) * k8[g0:g1].astype(np.float64).sum(axis=0) / n', 'kbar = float(k_scale[j]) * k8[g0:g1].astype(np.float64).sum(axis=0) / 32'),
 ('oracle/attention.py', 'vbar = v[g0:g1].mean(axis=0)', 'vbar = v[g0:g1].sum(axis=0) / 32'),
 ('oracle/attention.py', 'lg = (float(q_scale[i]) * scale) * (Qi @ kbar) + math.log(n)', 'lg = (float(q_scale[i]) * scale) * (Qi @ kbar) + math.log2(n)'),
 ('oracle/attention.py', 'logits.append((float(q_scale[i]) * float(k_scale[j]) * scale) * dots)\n                values', 'logits.append((float(q_scale[i]) * scale) * dots)\n                values'),
 ('oracle/attention.py', '            elif centroid_mode:', '            elif False:'),
 ('oracle/attention.py', 'return (e @ values) / l[:, None], m + np.log(l)', 'return (e @ values) / l[:, None], m + np.log2(l)'),
 ('oracle/attention.py', 'return 1.0 / math.sqrt(d) if', 'return 1.0 / d if'),
 ('oracle/attention.py', 'cols = np.arange(nKB) // 2', 'cols = np.minimum((np.arange(nKB) + 1) // 2, mask_bh.shape[1] - 1)'),
 ('oracle/attention.py', 'm[xq, xk] = 1 if fq - window <= fk <= fq else 0', 'm[xq, xk] = 1 if fq - window < fk <= fq else 0'),
 ('oracle/attention.py', 'fq = (128 * xq) // frame_tokens', 'fq = (128 * xq + 127) // frame_tokens'),
 ('oracle/attention.py', 'return sol_attention_head(q8, q_scale, k8, k_scale, v, allowed, 0,', 'return sol_attention_head(q8, q_scale, k8, k_scale, v, allowed, 1,'),
 ('oracle/attention.py', '            lse[r0:r1] = -math.inf\n            continue', '            lse[r0:r1] = 0.0\n            continue'),
 ('oracle/attention.py', '            logits.append((float(q_scale[i]) * float(k_scale[j]) * scale) * dots)\n            values.append(v[t0:t1])\n        for n, kbar', '            logits.append((float(q_scale[i]) * scale) * dots)\n            values.append(v[t0:t1])\n        for n, kbar'),
 ('oracle/attention.py', 'logits.append(((float(q_scale[i]) * scale) * (Qi @ kbar) + math.log(n))[:, None])', 'logits.append(((float(q_scale[i]) * scale) * (Qi @ kbar))[:, None])'),
 ('oracle/attention.py', 'for grp in table[j]]', 'for grp in table[j][:1]]'),
 ('oracle/attention.py', 'virtual = [grp for s in src_map for', 'virtual = [grp for s in sorted(set(src_map)) for'),
 ('oracle/attention.py', 'for j in range(s * bps, (s + 1) * bps)', 'for j in range(s * bps, (s + 1) * bps - 1)'),
 ('oracle/attention.py', 'for j in range(s * bps, (s + 1) * bps) for grp', 'for j in range((n_src - 1 - s) * bps, (n_src - s) * bps) for grp'),
 ('oracle/kv_cache.py', 'for t0, t1 in block_rows(k.shape[0], SLAB_ROWS):', 'for t0, t1 in block_rows(k.shape[0], 64):'),
 ('oracle/kv_cache.py', 'self.slabs.pop(0)', 'self.slabs.pop()'),
 ('oracle/kv_cache.py', 'logits.append((float(q_scale[i]) * float(s["k_scale"][b]) * scale) * dots)', 'logits.append((float(q_scale[i]) * float(s["k_scale"][0]) * scale) * dots)'),
 ('oracle/kv_cache.py', 'values.append(s["v8"][t0:t1].astype(np.float64) * float(s["v_scale"][b]))', 'values.append(s["v8"][t0:t1].astype(np.float64))'),
 ('oracle/kv_cache.py', '            if not mask[i, x]:', '            if not mask[i, len(cache.slabs) - 1 - x]:'),
 ('oracle/kv_cache.py', 'v8, vs = quantize_blocks(v[t0:t1], K_ROWS)', 'v8, vs = quantize_blocks(v[t0:t1], Q_ROWS)'),
 ('oracle/kv_cache.py', 'while len(self.slabs) > self.capacity:', 'while len(self.slabs) > self.capacity + 1:'),
]


def _copy_tree(dst: str) -> None:
    """The oracle, its pins and their imports, copied so that mutations never touch tracked files."""
    for d in ("oracle", "tests", "workloads"):
        shutil.copytree(os.path.join(ROOT, d), os.path.join(dst, d),
                        ignore=shutil.ignore_patterns("__pycache__", "*.pyc"))


def main() -> int:
    survivors, errors = [], []
    with tempfile.TemporaryDirectory(prefix="oracle_mut_") as tmp:
        _copy_tree(tmp)
        for f, old, new in M:
            path = os.path.join(tmp, f)
            src = open(path).read()
            if src.count(old) != 1:
                print("NO MATCH", f, old[:60])
                errors.append((f, new))
                continue
            open(path, "w").write(src.replace(old, new))
            try:
                r = subprocess.run([sys.executable, "-m", "pytest", *PINS, "-x", "-q", "-p", "no:cacheprovider"],
                                   cwd=tmp, capture_output=True, text=True, timeout=900)
                rc = r.returncode
            except subprocess.TimeoutExpired:
                rc = None
            finally:
                open(path, "w").write(src)
            # pytest exits 1 when tests ran and some failed: only that counts as caught. Exit 2-4
            # (interrupted, internal error, usage or collection error) and a timeout are errors.
            if rc == 1:
                verdict = "KILLED  "
            elif rc == 0:
                verdict = "SURVIVED"
                survivors.append((f, new))
            else:
                verdict = f"ERROR({rc})"
                errors.append((f, new))
            print(verdict, f, "|", " ".join(new.split())[:90], flush=True)
    caught = len(M) - len(survivors) - len(errors)
    print(f"{caught} of {len(M)} mutations caught by a failing pin; {len(survivors)} survived; "
          f"{len(errors)} errors (no match, collection error or timeout)")
    return 1 if survivors or errors else 0


if __name__ == "__main__":
    sys.exit(main())

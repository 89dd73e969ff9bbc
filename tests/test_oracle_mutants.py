"""The pins can fail: plausible mistakes, planted one at a time in a private copy of the oracle.

Each mutant below is a slip that a transcription of the pages could make (a dropped term, a wrong
sign or index, a swapped operand, a wrong rounding).  It is applied to a copy of oracle/ in a
temporary directory (oracle/ itself is never touched), and the oracle's pin suite
(test_oracle_pins.py) is run against that copy in a subprocess; every mutant must make at least one
pin fail, and the unmodified copy must pass.  CPU only, the copies run in parallel.
"""
import concurrent.futures
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# (what the mistake is, the oracle's text, the text with the mistake)
MUTANTS = [
    ('group score top-1 instead of top-2',
     'gscore = (top2[:, 0] + top2[:, 1]).astype(np.float32)',
     'gscore = top2[:, 0]'),
    ('bias enters weights',
     'wts[t] = gate_weights(s[t, e], hp.do_renorm, hp.route_scale)',
     'wts[t] = gate_weights(b[t, e], hp.do_renorm, hp.route_scale)'),
    ('no renorm',
     '    if do_renorm:\n        total',
     '    if False:\n        total'),
    ('ascending topk',
     'return np.argsort(-np.asarray(v), kind="stable")',
     'return np.argsort(np.asarray(v), kind="stable")[::-1]'),
    ('heaviest experts in greedy',
     'return np.argsort(f, kind="stable")[:k]',
     'return np.argsort(-f, kind="stable")[:k]'),
    ('greedy adds p not p/k',
     'f[chosen] += p[i] / k',
     'f[chosen] += p[i]'),
    ('silu wrong sign',
     'return z / (1.0 + np.exp(-z))',
     'return z / (1.0 + np.exp(z))'),
    ('w1/w3 swapped roles',
     'a = silu(zg) * zv',
     'a = silu(zv) * zg'),
    ('w2 output features reversed',
     'return round_bf16(h @ np.asarray(w2, np.float64).T)',
     'return round_bf16(h @ np.asarray(w2, np.float64).T[:, ::-1])'),
    ('shared dropped',
     '        y = (y + np.asarray(shared_out, np.float32)).astype(np.float32)',
     '        pass'),
    ('sigmoid sign',
     's = 1.0 / (1.0 + np.exp(-l))',
     's = 1.0 / (1.0 + np.exp(l))'),
    ('softplus no sqrt',
     's = np.sqrt(softplus)',
     's = softplus'),
    ('logit offset ignored',
     'l = (l + np.asarray(logit_offset, np.float32)).astype(np.float32)',
     'pass'),
    ('dispatch unstable',
     'slot_of_row = np.argsort(flat, kind="stable")',
     'slot_of_row = np.argsort(flat, kind="stable")[::-1]'),
    ('ngram swaps a and b',
     '[(a * int(q) + b) % n_experts for q in primes]',
     '[(b * int(q) + a) % n_experts for q in primes]'),
    ('ngram drops b',
     '[(a * int(q) + b) % n_experts for q in primes]',
     '[(a * int(q)) % n_experts for q in primes]'),
    ('bias update wrong sign',
     'bias[e] = np.float32(bias[e] - g)',
     'bias[e] = np.float32(bias[e] + g)'),
    ('bias update ignores k',
     'if counts[e] * E > T * k:',
     'if counts[e] * E > T:'),
    ('best keeps worst',
     'if best is None or mx < best[3]:',
     'if best is None or mx > best[3]:'),
    ('best keeps later tie',
     'if best is None or mx < best[3]:',
     'if best is None or mx <= best[3]:'),
    ('e2m1 exponent bias 0',
     'np.ldexp(1.0 + 0.5 * m, (e - 1).astype(np.int64))',
     'np.ldexp(1.0 + 0.5 * m, e.astype(np.int64))'),
    ('e2m1 subnormal 1.0',
     'np.where(e == 0, 0.5 * m,',
     'np.where(e == 0, 1.0 * m,'),
    ('mxfp4 nibble order',
     'codes[:, 0::2] = packed & 0xF\n    codes[:, 1::2] = packed >> 4',
     'codes[:, 0::2] = packed >> 4\n    codes[:, 1::2] = packed & 0xF'),
    ('ue8m0 bias 128',
     'np.ldexp(1.0, s - 127)',
     'np.ldexp(1.0, s - 128)'),
    ('clamp gate both sides',
     'zg = np.minimum(zg, limit)',
     'zg = np.clip(zg, -limit, limit)'),
    ('row weight after rounding',
     '        a = a * np.asarray(row_weight, np.float32).astype(np.float64)[:, None]\n    h = round_bf16(a)',
     '        a = round_bf16(a) * np.asarray(row_weight, np.float32).astype(np.float64)[:, None]\n    h = round_bf16(a)'),
    ('bf16 truncation',
     'return np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)',
     'return np.ldexp(np.trunc(np.ldexp(m, 8)), e - 8)'),
    ('route_scale dropped',
     'return (w * np.float32(route_scale)).astype(np.float32)',
     'return w'),
    ('group score sums top-2 without a bias',
     'gscore = per.max(axis=1)',
     'gscore = np.sort(per, axis=1)[:, ::-1][:, :2].sum(axis=1).astype(np.float32)'),
    ('softmax renormalised',
     'return self.score_func in ("sigmoid", "sqrtsoftplus")',
     'return True'),
    ('softmax not normalised',
     's = z / z.sum(axis=-1, keepdims=True)',
     's = z'),
    ('groups not limited',
     'masked[kept] = per[kept]',
     'masked[:] = per'),
    ('worst groups kept',
     'kept = np.sort(gorder[:n_limited_groups])',
     'kept = np.sort(gorder[-n_limited_groups:])'),
    ('top-k skips the best',
     'experts = order[:topk]',
     'experts = order[1:topk + 1]'),
    ('hash table columns reversed',
     'idx = tid2eid[np.asarray(token_ids, np.int64)].astype(np.int64)',
     'idx = tid2eid[np.asarray(token_ids, np.int64)].astype(np.int64)[:, ::-1]'),
    ('hash gate not renormalised',
     '              do_renorm: bool = True):\n    """Hash-routed gate',
     '              do_renorm: bool = False):\n    """Hash-routed gate'),
    ('logits rounded to bf16',
     'l = round_f32(np.asarray(x, np.float64) @ np.asarray(w_gate, np.float64).T)',
     'l = round_bf16(np.asarray(x, np.float64) @ np.asarray(w_gate, np.float64).T).astype(np.float32)'),
    ('value clamp one-sided',
     'zv = np.clip(zv, -limit, limit)',
     'zv = np.minimum(zv, limit)'),
    ('combine ignores weights',
     'term = o.astype(np.float32) if weights is None else (o.astype(np.float32) * weights[t, j]).astype(np.float32)',
     'term = o.astype(np.float32)'),
    ('offsets inclusive scan',
     'offsets = np.concatenate([[0], np.cumsum(counts)])',
     'offsets = np.concatenate([np.cumsum(counts), [flat.shape[0]]])'),
    ('tok_of_row is the slot',
     'return counts, offsets, row_of_slot, slot_of_row // k',
     'return counts, offsets, row_of_slot, slot_of_row'),
    ('bias update moves at balance',
     'elif counts[e] * E < T * k:',
     'else:'),
    ('primes from m, not above',
     '    q = m + 1\n',
     '    q = m\n'),
    ('h not rounded to bf16',
     '    h = round_bf16(a)\n',
     '    h = a\n'),
    ('output not cast to bf16',
     '    return round_bf16(y)\n',
     '    return y.astype(np.float64)\n'),
    ('ue8m0 255 finite',
     'return np.where(s == 255, np.nan, np.ldexp(1.0, s - 127))',
     'return np.ldexp(1.0, s - 127)'),
    ('e2m1 sign ignored',
     'sign = np.where(code & 8, -1.0, 1.0)',
     'sign = 1.0'),
    ('greedy visits ascending p',
     'visit = _descending(p) if order is None else np.asarray(order)',
     'visit = _descending(-p) if order is None else np.asarray(order)'),
    ('e4m3 exponent bias 8',
     'np.ldexp(1.0 + m / 8.0, (e - 7).astype(np.int64))',
     'np.ldexp(1.0 + m / 8.0, (e - 8).astype(np.int64))'),
    ('e4m3 subnormal scale',
     'mag = np.where(e == 0, np.ldexp(m / 8.0, -6),',
     'mag = np.where(e == 0, np.ldexp(m / 8.0, -7),'),
    ('mx scale from 256, not 448',
     'e = np.where(np.ldexp(448.0, e) >= amax, e, e + 1)',
     'e = np.where(np.ldexp(256.0, e) >= amax, e, e + 1)'),
    ('mx scale saturating (floor)',
     'e = np.where(np.ldexp(448.0, e) >= amax, e, e + 1)',
     'e = e'),
    ('mx scale one too large',
     'e = np.where(np.ldexp(448.0, e) >= amax, e, e + 1)',
     'e = np.where(np.ldexp(448.0, e) >= amax, e, e + 1) + 1'),
    ('e4m3 ties away from zero',
     'pick = np.where(d_lo < d_hi, lo, np.where(d_hi < d_lo, hi, np.where(lo % 2 == 0, lo, hi)))',
     'pick = np.where(d_lo < d_hi, lo, hi)'),
    ('e4m3 truncates',
     'pick = np.where(d_lo < d_hi, lo, np.where(d_hi < d_lo, hi, np.where(lo % 2 == 0, lo, hi)))',
     'pick = lo'),
    ('mx blocks down columns',
     '    blocks = v.reshape(R, K // block, block)\n',
     '    blocks = v.T.reshape(K, R // block, block).transpose(1, 0, 2).reshape(R, K // block, block)\n'),
    ('mx h not quantised',
     '    hq = e4m3_block_dequant(*quantize_e4m3_block(act))\n',
     '    hq = act\n'),
]


def _pin_suite_on_copy(workdir: str, name: str, old: str, new: str) -> int:
    """pytest's exit status for the pin suite run against a copy of the oracle with `old` -> `new`."""
    d = os.path.join(workdir, name.replace(" ", "_").replace("/", "_"))
    shutil.copytree(os.path.join(ROOT, "oracle"), os.path.join(d, "oracle"),
                    ignore=shutil.ignore_patterns("__pycache__"))
    path = os.path.join(d, "oracle", "moe_oracle.py")
    with open(path) as f:
        src = f.read()
    if old:
        assert src.count(old) == 1, name
        src = src.replace(old, new)
    with open(path, "w") as f:
        f.write(src)
    os.makedirs(os.path.join(d, "tests"))
    for fn in ("test_oracle_pins.py", "conftest.py"):
        shutil.copy(os.path.join(ROOT, "tests", fn), os.path.join(d, "tests", fn))
    os.symlink(os.path.join(ROOT, "tests", "golden"), os.path.join(d, "tests", "golden"))
    os.symlink(os.path.join(ROOT, "mixture_experts_routing_gate_b200"),
               os.path.join(d, "mixture_experts_routing_gate_b200"))
    r = subprocess.run([sys.executable, "-m", "pytest", "tests/test_oracle_pins.py", "-x", "-q",
                        "-p", "no:cacheprovider"], cwd=d, capture_output=True, text=True, timeout=600)
    return r.returncode


@pytest.mark.slow
def test_every_planted_mistake_fails_a_pin(tmp_path):
    jobs = [("unmodified", "", "")] + MUTANTS
    workers = max(1, min(8, os.cpu_count() or 1))
    with concurrent.futures.ThreadPoolExecutor(max_workers=workers) as ex:
        codes = list(ex.map(lambda j: _pin_suite_on_copy(str(tmp_path), *j), jobs))
    status = dict(zip((j[0] for j in jobs), codes))
    assert status.pop("unmodified") == 0, "the unmodified copy of the oracle fails its pins"
    missed = [name for name, rc in status.items() if rc != 1]
    assert not missed, f"no pin fails for: {missed}"

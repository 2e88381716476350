"""Plant plausible mistakes in a copy of the oracle; some pin must catch each.

Each mutation rewrites one expression of ``oracle/attention.py`` (a dropped
term, a wrong sign or index, a swapped operand), loads the result as a fresh
module on the CPU and runs the pins against it.  The real oracle is not
touched.
"""
import importlib.util
import os
import sys
import types

import pytest

from oracle_pins import ALL_PINS

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle",
                   "attention.py")

MUTATIONS = [
    ("gqa head index", "return h_q // (Hq // Hkv)", "return h_q % Hkv"),
    ("strict causal", "return k_pos[None, :] <= q_pos[:, None]", "return k_pos[None, :] < q_pos[:, None]"),
    ("reversed causal", "return k_pos[None, :] <= q_pos[:, None]", "return k_pos[None, :] >= q_pos[:, None]"),
    ("cache_idx ignored", "base = 0 if cache_idx < 0 else int(cache_idx)", "base = 0"),
    ("scale dropped", "s = scale * (q[b, r, h, :] @ k[b, :n_keys, hk, :].T)", "s = (q[b, r, h, :] @ k[b, :n_keys, hk, :].T)"),
    ("no normalisation", "o[has] = (w[has] @ v[b, :n_keys, hk, :]) / l[has, None]", "o[has] = (w[has] @ v[b, :n_keys, hk, :])"),
    ("k used as v", "o[has] = (w[has] @ v[b, :n_keys, hk, :]) / l[has, None]", "o[has] = (w[has] @ k[b, :n_keys, hk, :]) / l[has, None]"),
    ("lse drops max", "has, m + np.log(np.where(has, l, 1.0)), NEG_INF)", "has, np.log(np.where(has, l, 1.0)), NEG_INF)"),
    ("rescale of l dropped", "l[b, h] = alpha * l[b, h] + p.sum(axis=1)", "l[b, h] = l[b, h] + p.sum(axis=1)"),
    ("rescale of acc dropped", "acc[b, h] = alpha[:, None] * acc[b, h] + p @ vc[b, :, hk, :]", "acc[b, h] = acc[b, h] + p @ vc[b, :, hk, :]"),
    ("rescale sign", "alpha = np.exp(m[b, h] - base)", "alpha = np.exp(base - m[b, h])"),
    ("block k offset dropped", "k_off + np.arange(Lk, dtype=np.int64)", "np.arange(Lk, dtype=np.int64)"),
    ("block q offset dropped", "_visible(q_off + np.arange(Lq", "_visible(np.arange(Lq"),
    ("block scale dropped", "s = scale * (q[b, :, h, :] @ kc[b, :, hk, :].T)", "s = (q[b, :, h, :] @ kc[b, :, hk, :].T)"),
    ("finalize lse drops m", "lse = np.where(has, m + np.log(safe), NEG_INF)", "lse = np.where(has, np.log(safe), NEG_INF)"),
    ("ring direction ignored", "return (i + direction * s) % P", "return (i + s) % P"),
    ("ring always forward from 0", "return (i + direction * s) % P", "return s % P"),
    ("merge weight sign", "w = np.exp(L - base[None])", "w = np.exp(base[None] - L)"),
    ("merge lse drops max", "lse = np.where(has, base + np.log(safe), NEG_INF)", "lse = np.where(has, np.log(safe), NEG_INF)"),
    ("merge unweighted", "out = (w_t * o).sum(axis=0) /", "out = o.sum(axis=0) /"),
    ("softmax base", "w = np.exp(s - base[:, None])", "w = np.exp(s - base[:, None] - 1.0)"),
    ("bwd D term dropped", "ds = p * (dp - D[:, None])", "ds = p * dp"),
    ("bwd dv transposed", "dv[b, :, hk, :] += p.T @ do[b, :, h, :]", "dv[b, :, hk, :] += p.T @ q[b, :, h, :]"),
    ("bwd dk scale dropped", "dk[b, :, hk, :] += scale * (ds.T @ q[b, :, h, :])", "dk[b, :, hk, :] += (ds.T @ q[b, :, h, :])"),
    ("bwd dq uses v", "dq[b, :, h, :] = scale * (ds @ k[b, :, hk, :])", "dq[b, :, h, :] = scale * (ds @ v[b, :, hk, :])"),
    ("bwd group not summed", "dk[b, :, hk, :] += scale", "dk[b, :, hk, :] = scale"),
    ("bwd visit drops delta", "ds = p * (dp - delta[b, h][:, None])", "ds = p * dp"),
    ("bwd visit lse sign", "np.exp(np.where(live, s, 0.0) - base[:, None])",
     "np.exp(np.where(live, s, 0.0) + base[:, None])"),
    ("bwd visit dq unscaled", "dq[b, :, h, :] += scale * (ds @ kc[b, :, hk, :])",
     "dq[b, :, h, :] += (ds @ kc[b, :, hk, :])"),
    ("bwd visit dq overwritten", "dq[b, :, h, :] += scale * (ds @ kc[b, :, hk, :])",
     "dq[b, :, h, :] = scale * (ds @ kc[b, :, hk, :])"),
    ("bwd ring wrong kv chunk", "ks = slice(j * L, (j + 1) * L)", "ks = slice(i * L, (i + 1) * L)"),
    ("e4m3 exponent bias 8", "np.ldexp(1.0 + m / 8.0, e - 7)", "np.ldexp(1.0 + m / 8.0, e - 8)"),
    ("e4m3 subnormal as 2^-7", "np.ldexp(m / 8.0, -6)", "np.ldexp(m / 8.0, -7)"),
    ("e4m3 sign dropped", "return (sign * mag)[", "return (mag)["),
    ("e4m3 mantissa step 1/16", "(1.0 + m / 8.0, e - 7)", "(1.0 + m / 16.0, e - 7)"),
    ("fp8 v scaled by k_scale", "v = decode_e4m3(_u8(v8)) * vs[", "v = decode_e4m3(_u8(v8)) * ks["),
    ("fp8 scale transposed", "k = decode_e4m3(_u8(k8)) * ks[:, None, :, None]",
     "k = decode_e4m3(_u8(k8)) * ks.T[:, None, :, None]"),
    ("window one key short", "(kp >= np.maximum(0, qp - window))", "(kp > np.maximum(0, qp - window))"),
    ("window not causal", "vis = (kp <= qp) & (kp >= np.maximum", "vis = (kp <= qp + 1) & (kp >= np.maximum"),
    ("anchor minus one dropped", "vis |= (a > 0) & (kp == a - 1)", "vis |= (a > 0) & (kp == a)"),
    ("future anchor one early", "vis |= (a < n - anchor_period) & (kp == a + anchor_period)",
     "vis |= (a < n - anchor_period) & (kp == a + anchor_period - 1)"),
    ("anchor not floored", "a = (qp // anchor_period) * anchor_period", "a = qp // anchor_period"),
    ("bwd visit dk from dout", "dk[b, :, hk, :] += scale * (ds.T @ q[b, :, h, :])",
     "dk[b, :, hk, :] += scale * (ds.T @ do[b, :, h, :])"),
    # The row-block loop of attention_ref (several blocks, sampled rows and
    # heads, and key rows long enough to shrink the block).
    ("row block out written at 0", "out[b, r0:r0 + r.shape[0], hi, :] = o", "out[b, :r.shape[0], hi, :] = o"),
    ("row block lse written at 0", "lse[b, hi, r0:r0 + r.shape[0]] = np.where(\n",
     "lse[b, hi, :r.shape[0]] = np.where(\n"),
    ("key bound from the block's last row", "min(N_kv, qp.max() + 1)", "min(N_kv, qp[-1] + 1)"),
    ("sample positions by block index", "qp = pos_all[r]", "qp = pos_all[r0:r0 + r.shape[0]]"),
    ("sampled heads taken in sorted order", "        for hi, h in enumerate(heads):\n            hk = _kv_head(h, Hq, Hkv)\n"
     "            # Bound", "        for hi, h in enumerate(sorted(heads)):\n            hk = _kv_head(h, Hq, Hkv)\n"
     "            # Bound"),
    ("long rows lose the last key", "n_keys = N_kv if not causal else int(min(N_kv, qp.max() + 1))",
     "n_keys = N_kv if not causal else int(min(N_kv - (N_kv > 131072), qp.max() + 1))"),
]


def _load_mutant(old, new):
    text = open(SRC).read()
    assert text.count(old) >= 1, f"mutation anchor not found: {old!r}"
    text = text.replace(old, new)
    mod = types.ModuleType("oracle_mutant")
    mod.__file__ = SRC
    exec(compile(text, SRC + ":mutant", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_mutation_is_caught(name, old, new):
    mutant = _load_mutant(old, new)
    # The pins run cheapest first; the first one that fails is enough.
    caught = None
    for pin in ALL_PINS:
        try:
            pin(mutant)
        except Exception as e:  # AssertionError or numerical breakage
            caught = f"{pin.__name__}: {type(e).__name__}"
            break
    assert caught, f"mutation '{name}' passed every pin"

"""Plants one plausible mistake at a time in a copy of the oracle and checks that
the pins catch it.  The mistakes are edits of the oracle's own source text, made
on the CPU; the real module is never touched."""
import importlib.util
import inspect
import types

import pytest

import oracle_pins
from oracle import flce_oracle

# (description, original text, mutated text); each original must occur in the source.
MUTATIONS = [
    ("one-hot added instead of subtracted", "G[rows, yv] -= 1.0                            # minus the one-hot",
     "G[rows, yv] += 1.0                            # minus the one-hot"),
    ("ignored rows not masked in G", "    return np.where(valid, s, 0.0)", "    return s"),
    ("mean over all rows, not valid rows", 's = np.full(valid.shape, (1.0 / n) if n else 0.0)',
     's = np.full(valid.shape, (1.0 / valid.size) if n else 0.0)'),
    ("per-row upstream weights ignored", "G *= s[:, None]                               # s_i",
     "G *= s[:, None] ** 0 * s[0]                   # s_i"),
    ("softmax not normalised", "G = np.exp(Z - lse[:, None])                  # softmax",
     "G = np.exp(Z)                                 # softmax"),
    ("max dropped from log-sum-exp", "return m + np.log(np.exp(Z - m[:, None]).sum(axis=1))",
     "return np.log(np.exp(Z - m[:, None]).sum(axis=1))"),
    ("target logit added to the row loss",
     "row_loss = np.where(valid, lse - Z[rows, yv], 0.0)\n    loss = float((s * row_loss).sum())           # mean",
     "row_loss = np.where(valid, lse + Z[rows, yv], 0.0)\n    loss = float((s * row_loss).sum())           # mean"),
    ("dW from X transposed against G", "dW = G.T @ X", "dW = (X.T @ G).T * 0 + G.T @ (X * 0.5)"),
    ("dX against the wrong operand", "dX = G @ W", "dX = G @ (W - W.mean(axis=0)) * 0.5"),
    ("full-size loss drops the target logit", "row_loss = np.where(valid, lse - zy, 0.0)",
     "row_loss = np.where(valid, lse, 0.0)"),
    ("full-size dW one-hot sign", "G -= (y[:, None] == J[None, :])", "G += (y[:, None] == J[None, :])"),
    ("full-size dX ignores the valid mask", "    G *= valid[:, None]\n    G *= (1.0 / n) if n else 0.0\n    return G @ W64",
     "    G *= (1.0 / n) if n else 0.0\n    return G @ W64"),
    ("logit CE: one-hot sign", "    G[rows, yv] -= 1.0\n    G *= s[:, None]\n    return loss, G, lse, n, row_loss",
     "    G[rows, yv] += 1.0\n    G *= s[:, None]\n    return loss, G, lse, n, row_loss"),
    ("logit CE: row loss without the target logit", "    row_loss = np.where(valid, lse - Z[rows, yv], 0.0)\n    loss = float((s * row_loss).sum())\n    G = np.exp(Z - lse[:, None])\n    G[rows, yv] -= 1.0\n    G *= s[:, None]\n    return loss, G",
     "    row_loss = np.where(valid, lse, 0.0)\n    loss = float((s * row_loss).sum())\n    G = np.exp(Z - lse[:, None])\n    G[rows, yv] -= 1.0\n    G *= s[:, None]\n    return loss, G"),
    ("target range not checked", "bad = valid & ((y < 0) | (y >= V))", "bad = valid & (y < -10**9)"),
    ("shard target not shifted by the shard start", "    local = y - v0\n", "    local = y\n"),
    ("shard target past the shard's end accepted", "(local < Ws.shape[0])", "(local <= Ws.shape[0])"),
    ("shards merged by max instead of log-sum-exp", "return log_sum_exp(L.T), _f64(all_zy).sum(axis=0)",
     "return L.max(axis=0), _f64(all_zy).sum(axis=0)"),
    ("shard target logits averaged", "return log_sum_exp(L.T), _f64(all_zy).sum(axis=0)",
     "return log_sum_exp(L.T), _f64(all_zy).mean(axis=0)"),
    ("blocked lse drops the ragged last block", "    for b in range(0, X.shape[0], block):",
     "    out[:] = 0.0\n    for b in range(0, X.shape[0] - X.shape[0] % block, block):"),
    ("blocked loss divides by all rows", "loss = float(row_loss.sum() / n) if n else 0.0",
     "loss = float(row_loss.sum() / len(y)) if n else 0.0"),
    ("dX rows take another row's log-sum-exp", "G = np.exp(Z - np.asarray(lse_rows, dtype=np.float64)[:, None])",
     "G = np.exp(Z - np.asarray(lse_rows, dtype=np.float64)[::-1][:, None])"),
    ("dW rows keep ignored rows", "    G *= valid[:, None]\n    G *= (1.0 / n) if n else 0.0\n    return G.T @ X64",
     "    G *= (1.0 / n) if n else 0.0\n    return G.T @ X64"),
    ("blocked gradients drop the ragged last block", "    for b0 in range(0, N, block):",
     "    for b0 in range(0, N - N % block, block):"),
    ("blocked G keeps ignored rows", "Z *= (vb * inv_n)[:, None]", "Z *= inv_n"),
    ("blocked dW takes the first block's rows of X", "dW += Z.T @ X64[b0:b1]", "dW += Z.T @ X64[:b1 - b0]"),
    ("blocked one-hot added", "Z[rows, yb] -= 1.0", "Z[rows, yb] += 1.0"),
    ("blocked loss over all rows' count", "    loss = float(loss_sum / n) if n else 0.0",
     "    loss = float(loss_sum / N) if n else 0.0"),
    ("pair loss: sign of the margin", "    loss = float(np.logaddexp(0.0, -m).sum() / P)",
     "    loss = float(np.logaddexp(0.0, m).sum() / P)"),
    ("pair loss: rejected gradient added", "        grad[r[k]] -= beta * gm[k]", "        grad[r[k]] += beta * gm[k]"),
    ("pair loss: ignored rows weighted", "    w[y == ignore_index] = 0.0\n", "    pass\n"),
    ("pair loss: reference log-probs added", "d = logp if ref_logp is None else logp - _f64(ref_logp)",
     "d = logp if ref_logp is None else logp + _f64(ref_logp)"),
    ("bf16 tensors converted through fp16", "            a = a.float()", "            a = a.half().float()"),
]


def _mutant(orig, new):
    src = inspect.getsource(flce_oracle)
    assert src.count(orig) == 1, f"mutation anchor not unique/present: {orig!r}"
    mod = types.ModuleType("flce_oracle_mutant")
    exec(compile(src.replace(orig, new), "<mutant>", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("desc,orig,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_mutant(desc, orig, new):
    mod = _mutant(orig, new)
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(mod)
        except Exception as e:  # AssertionError, or a crash the mistake causes
            caught.append(f"{pin.__name__}: {type(e).__name__}")
    assert caught, f"no pin caught the planted mistake: {desc}"

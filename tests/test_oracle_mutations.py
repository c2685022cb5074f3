"""The oracle's pins against planted mistakes.

Each case rewrites one line of an oracle function on the CPU (a sign, an index, a dropped
term, a transposed operand, a different rounding or placement rule), installs the mutant
for the duration of the test, and runs the pins of `test_oracle_pins.py` and
`test_placement_oracle.py`. At least one pin must fail for every mutant; otherwise that
slip would go unnoticed in the reference the CUDA path is compared against.
"""
import inspect
import textwrap

import pytest

import test_oracle_pins as PINS
import test_placement_oracle as PPINS
from oracle import dkv_oracle as O
from oracle import placement as PL


def _pins():
    runs = []
    for name, fn in sorted(vars(PINS).items()):
        if not name.startswith("test_") or not callable(fn):
            continue
        params = inspect.signature(fn).parameters
        if "layout" in params:
            runs += [(f"{name}[{lay}]", (lambda f=fn, l=lay: f(l))) for lay in (0, 1)]
        else:
            runs.append((name, fn))
    return runs


def _placement_pins():
    runs = []
    for name, fn in sorted(vars(PPINS).items()):
        if not name.startswith("test_") or not callable(fn):
            continue
        params = inspect.signature(fn).parameters
        if "budget" in params:
            runs += [(f"{name}[{b}]", (lambda f=fn, b=b: f(0, b))) for b in (0, 3, 20)]
        else:
            runs.append((name, fn))
    return runs


def _mutant(fn, old, new, namespace):
    src = textwrap.dedent(inspect.getsource(fn))
    assert src.count(old) >= 1, f"mutation site not found: {old!r}"
    ns = dict(namespace)
    exec(compile(src.replace(old, new), f"<mutant of {fn.__name__}>", "exec"), ns)
    return ns[fn.__name__]


def _failing(runs):
    failed = []
    for name, run in runs:
        try:
            run()
        except Exception:  # an assertion, or a crash the mutant causes
            failed.append(name)
    return failed


# (case, function, original text, mutated text)
ORACLE_MUTANTS = [
    ("rope-sign", "rope_rotate_half", "[a * c - b * s, b * c + a * s]", "[a * c + b * s, b * c - a * s]"),
    ("rope-adjacent-pairs", "rope_rotate_half", "a, b = vec[..., :half], vec[..., half:]",
     "a, b = vec[..., 0::2], vec[..., 1::2]"),
    ("rope-frequency-exponent", "rope_rotate_half", "-2.0 * i / D", "-1.0 * i / D"),
    ("rope-position-offset", "rope_rotate_half", "ang = float(pos) * inv", "ang = float(pos + 1) * inv"),
    ("softmax-no-scale", "softmax_attention", "s = (K @ q) / math.sqrt(D)", "s = K @ q"),
    ("softmax-scale-by-D", "softmax_attention", "s = (K @ q) / math.sqrt(D)", "s = (K @ q) / D"),
    ("gqa-h-mod-g", "decode_step", "h // G", "h % G"),
    ("drop-new-key-value", "decode_step",
     "Kf = np.concatenate([Kc, bf16_to_f64(k_hat[b, g])[None]], axis=0)", "Kf = Kc"),
    ("new-key-unrounded", "decode_step", "bf16_to_f64(k_hat[b, g])[None]", "k_rot[g][None]"),
    ("new-value-unrounded", "decode_step", "bf16_to_f64(v_hat[b, g])[None]", "v[g][None]"),
    ("new-key-not-rotated", "decode_step", "k_hat[b] = f64_to_bf16_rne(k_rot)", "k_hat[b] = f64_to_bf16_rne(k)"),
    ("rope-position-of-last-cached", "decode_step", "q_rot = rope_rotate_half(q, ctx, theta)",
     "q_rot = rope_rotate_half(q, max(ctx - 1, 0), theta)"),
    ("split-k-takes-v-rows", "split_qkv", "k = qkv[Hq * D: (Hq + Hkv) * D]",
     "k = qkv[(Hq + Hkv) * D: (Hq + 2 * Hkv) * D]"),
    ("projection-transposed", "qkv_projection", "np.asarray(W, dtype=np.float64) @",
     "np.asarray(W, dtype=np.float64).T @"),
    ("rounding-half-up", "f64_to_bf16_rne", "np.rint(scaled)", "np.floor(scaled + 0.5)"),
    ("rounding-truncate", "f64_to_bf16_rne", "np.rint(scaled)", "np.trunc(scaled)"),
    ("rounding-one-bit-more", "f64_to_bf16_rne", "e - 8", "e - 9"),
    ("rounding-via-fp32", "f64_to_bf16_rne", "x = np.asarray(x, dtype=np.float64)",
     "x = np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)"),
    ("chunk-kv-head-swapped", "chunk_view", "return tier[layer, phys, kv, g]", "return tier[layer, phys, g, kv]"),
    ("gather-ignores-tier", "gather_sequence", "chunk_view(tiers[t], layout, layer, ids[sel], 0, g)",
     "chunk_view(tiers[0], layout, layer, ids[sel] % max(tiers[0].shape[1], 1), 0, g)"),
    ("gather-off-by-one", "gather_sequence", "K.reshape(nb * T, D)[:ctx]", "K.reshape(nb * T, D)[1:ctx + 1]"),
    ("layout-reshape-not-transpose", "layer_first_to_page_first",
     "out[:, l] = pool[l]", "out.reshape((L, P) + pool.shape[2:])[l] = pool[l]"),
    ("gemm-wrong-index", "gemm_entries", "bf16_to_f64(Bt_bits[int(j)])", "bf16_to_f64(Bt_bits[int(i) % len(Bt_bits)])"),
    ("gemm-bound-keeps-sign-of-a", "gemm_abs_bound", "np.abs(bf16_to_f64(A_bits[int(i)]))",
     "bf16_to_f64(A_bits[int(i)])"),
    ("gemm-bound-keeps-sign-of-b", "gemm_abs_bound", "np.abs(bf16_to_f64(Bt_bits[int(j)]))",
     "bf16_to_f64(Bt_bits[int(j)])"),
    ("gemm-bound-wrong-column", "gemm_abs_bound", "np.abs(bf16_to_f64(Bt_bits[int(j)]))",
     "np.abs(bf16_to_f64(Bt_bits[int(i) % len(Bt_bits)]))"),
]


@pytest.mark.parametrize("case,fname,old,new", ORACLE_MUTANTS, ids=[m[0] for m in ORACLE_MUTANTS])
def test_oracle_pins_catch_planted_mistake(case, fname, old, new, monkeypatch):
    monkeypatch.setattr(O, fname, _mutant(getattr(O, fname), old, new, vars(O)))
    assert _failing(_pins()), f"no pin fails with the planted mistake {case}"


PLACEMENT_MUTANTS = [
    ("demote-newest", "_demote_oldest", "j = next(k for k, (t, _) in enumerate(self.blocks[r]) if t == HBM)",
     "j = max(k for k, (t, _) in enumerate(self.blocks[r]) if t == HBM)"),
    ("promote-oldest", "_promote_newest", "j = max(k for k, (t, _) in enumerate(self.blocks[r]) if t == HOST)",
     "j = next(k for k, (t, _) in enumerate(self.blocks[r]) if t == HOST)"),
    ("window-ignores-new-row", "add", "W = self.budget // (self.n() + 1)", "W = self.budget // max(self.n(), 1)"),
    ("largest-free-id", "_take", "i = min(self.free[tier])", "i = max(self.free[tier])"),
    ("new-block-always-host", "step", "tier = HBM if W >= 1 else HOST", "tier = HOST"),
    ("no-slot-for-new-token", "nb", "return length // self.T + 1", "return max((length + self.T - 1) // self.T, 1)"),
    ("moved-row-not-rewritten", "remove",
     "self._dirty.update((r, j) for j in range(len(self.blocks[r])))", "pass"),
]


@pytest.mark.parametrize("case,meth,old,new", PLACEMENT_MUTANTS, ids=[m[0] for m in PLACEMENT_MUTANTS])
def test_placement_pins_catch_planted_mistake(case, meth, old, new, monkeypatch):
    fn = getattr(PL.RecencyPlacement, meth)
    monkeypatch.setattr(PL.RecencyPlacement, meth, _mutant(fn, old, new, vars(PL)))
    assert _failing(_placement_pins()), f"no pin fails with the planted mistake {case}"


def test_unmutated_pins_pass():
    assert _failing(_pins()) == []
    assert _failing(_placement_pins()) == []

"""The pins must catch plausible mistakes: plant one mistake at a time in a copy of the
oracle (CPU only), run the pins against the copy, and require at least one to fail."""
import importlib.util
import os
import sys

import pytest

import test_oracle_pins as P

ORACLE_SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                          "oracle", "awq_oracle.py")

# (name, text in the oracle, planted replacement)
MUTATIONS = [
    ("divisor_16", "(mx - mn) / np.float32(QMAX)", "(mx - mn) / np.float32(16)"),
    ("no_fp16_scale", "scale16 = fp16_rn(scale32)\n        sc = scale16.astype(np.float32)\n        zero",
     "scale16 = fp16_rn(scale32)\n        sc = scale32\n        zero"),
    ("round_half_up", "q = np.clip(np.rint(g / sc[:, :, None]) + zero",
     "q = np.clip(np.floor(g / sc[:, :, None] + 0.5) + zero"),
    ("zero_sign", "np.rint(-mn / sc)", "np.rint(mn / sc)"),
    ("zero_floor", "np.rint(-mn / sc)", "np.floor(-mn / sc)"),
    ("sym_divisor_8", "amax / np.float32(7)", "amax / np.float32(8)"),
    ("sym_offset", "np.clip(np.rint(g / sc[:, :, None]), -8, 7) + 8", "np.clip(np.rint(g / sc[:, :, None]), -8, 7) + 7"),
    ("no_scale_s", "ws = w32 * s32[None, :]", "ws = w32"),
    ("pack_reversed", "out |= p[:, :, j] << np.uint32(4 * j)", "out |= p[:, :, j] << np.uint32(28 - 4 * j)"),
    ("code_order_plain", "CODE_NIBBLE = (0, 4, 1, 5, 2, 6, 3, 7)", "CODE_NIBBLE = (0, 1, 2, 3, 4, 5, 6, 7)"),
    ("code_order_swapped", "CODE_NIBBLE = (0, 4, 1, 5, 2, 6, 3, 7)", "CODE_NIBBLE = (4, 0, 5, 1, 6, 2, 7, 3)"),
    ("absmean_no_abs", "X = np.abs(np.asarray(X16", "X = (np.asarray(X16"),
    ("absmean_divide_K", "/ np.float64(X.shape[0])", "/ np.float64(X.shape[1])"),
    ("alpha_endpoint", "np.arange(n_grid, dtype=np.float64) / np.float64(n_grid)",
     "np.arange(n_grid, dtype=np.float64) / np.float64(n_grid - 1)"),
    ("pow_via_f32", "p = np.power(np.asarray(m, dtype=np.float64), np.float64(alpha))",
     "p = np.power(np.asarray(m, dtype=np.float32), np.float32(alpha)).astype(np.float64)"),
    ("dequant_no_zero", "return ((q - z[:, :, None]) * sc[:, :, None]).reshape(N, K)",
     "return (q * sc[:, :, None]).reshape(N, K)"),
    ("linear_transposed", "return X @ deq.T", "return (deq @ X.T).T * 1.0000001"),
    ("loss_no_inverse_s", "dW = deq / s[None, :] - np.asarray", "dW = deq - np.asarray"),
    ("loss_sign", "dW = deq / s[None, :] - np.asarray(W16, dtype=np.float16).astype(np.float64)",
     "dW = deq / s[None, :] + np.asarray(W16, dtype=np.float16).astype(np.float64)"),
    ("argmax", "best = int(np.argmin(losses))", "best = int(np.argmax(losses))"),
    ("argmin_last", "best = int(np.argmin(losses))", "best = int(len(losses) - 1 - np.argmin(losses[::-1]))"),
    ("fold_multiply", "return fp16_rn(X / s[None, :])", "return fp16_rn(X * s[None, :])"),
    ("fp16_via_f32", "return np.asarray(x).astype(np.float16)",
     "return np.asarray(x).astype(np.float32).astype(np.float16)"),
    ("wmean_no_abs", "Wa = np.abs(np.asarray(W16", "Wa = (np.asarray(W16"),
    ("duo_weight_exponent_alpha", "np.float64(1.0) - np.float64(alpha)", "np.float64(alpha)"),
    ("duo_multiply", "np.minimum(np.maximum(a / b, S_MIN), S_MAX)", "np.minimum(np.maximum(a * b, S_MIN), S_MAX)"),
    ("duo_no_cap", "np.minimum(np.maximum(a / b, S_MIN), S_MAX)", "np.maximum(a / b, S_MIN)"),
    ("duo_argmax", "top = int(np.argmin(losses))", "top = int(np.argmax(losses))"),
    ("clip_ratio_sign", "np.float64(1.0) - j / np.float64(n_grid)", "np.float64(1.0) + j / np.float64(n_grid)"),
    ("clip_no_fp32_ratio", "c = (np.asarray(ratio, dtype=np.float32) * amax).astype(np.float32)",
     "c = (np.asarray(ratio, dtype=np.float64) * 0.999 * amax).astype(np.float32)"),
    ("clip_reference_clipped", "dW = deq / s[None, :] - Wd",
     "dW = deq / s[None, :] - (clip_groups(g, r).reshape(N, K) / s[None, :])"),
    ("clip_argmax", "idx = np.argmin(err, axis=2)", "idx = np.argmax(err, axis=2)"),
    ("clip_group_transposed", "E = X[:, gi * G:(gi + 1) * G] @ dW[:, gi * G:(gi + 1) * G].T",
     "E = X[:, gi * G:(gi + 1) * G] @ dW[:, gi * G:(gi + 1) * G][:, ::-1].T"),
]

PIN_NAMES = [n for n in dir(P) if n.startswith("test_")]


def _load_mutant(src: str):
    spec = importlib.util.spec_from_loader("awq_oracle_mutant", loader=None)
    mod = importlib.util.module_from_spec(spec)
    exec(compile(src, "awq_oracle_mutant.py", "exec"), mod.__dict__)
    return mod


def _run_all_pins(mutant) -> list:
    """Names of pins that fail against the mutant."""
    import inspect
    import json
    failed = []
    saved = P.O
    P.O = mutant
    try:
        for name in PIN_NAMES:
            fn = getattr(P, name)
            params = inspect.signature(fn).parameters
            calls = [{}]
            if "case" in params:
                cases = json.load(open(os.path.join(P.GOLDEN, "handworked_groups.json")))["cases"]
                calls = [{"case": c} for c in cases]
            if "G" in params and "zp" in params:
                calls = [{"G": 64, "zp": True}, {"G": 128, "zp": False}]
            elif "zp" in params:
                calls = [{"zp": True}, {"zp": False}]
            for kw in calls:
                try:
                    fn(**kw)
                except Exception:        # an assertion or an error both count as caught
                    failed.append(name)
                    break
    finally:
        P.O = saved
    return failed


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(name, old, new):
    src = open(ORACLE_SRC).read()
    assert src.count(old) == 1, f"mutation anchor not found once: {old!r}"
    mutant = _load_mutant(src.replace(old, new))
    failed = _run_all_pins(mutant)
    assert failed, f"no pin caught the planted mistake {name}"

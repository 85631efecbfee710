"""Mutation audit of the oracle's pins (CPU; not collected by pytest, ~4 minutes).

Plants one plausible slip at a time in a copy of ``oracle/svdq_oracle.py`` (a
wrong constant, sign, tie rule, operand, axis, rounding step or segment bound)
and runs the oracle's CPU pins (``tests/test_oracle_*.py``) against the copy.
Every slip must make at least one pin fail.  Run:

    python tests/oracle_mutation_audit.py

It prints one line per slip and exits 1 if any slip passes the pins.  Replacing
a value beyond 6 by 6 before the E2M1 rounding is not listed: the nearest-value
search already clips there, so that change computes the same function.
"""
import os
import shutil
import subprocess
import sys
import tempfile

REPO = os.path.abspath(os.path.join(os.path.dirname(__file__), ".."))
SRC = os.path.join(REPO, "oracle", "svdq_oracle.py")
# (slip, text of the oracle it replaces, replacement)
M = [
    ("scale divisor 4 instead of 6", "d = np.float32(np.float32(6.0) * s_g)", "d = np.float32(np.float32(4.0) * s_g)"),
    ("smoothing multiplies by lambda", "xs = xf * np.asarray(inv_lambda, dtype=np.float32)[None, :]", "xs = xf / np.asarray(inv_lambda, dtype=np.float32)[None, :]"),
    ("group absmax without abs", "a = np.abs(blocks).max(axis=2)", "a = np.maximum(blocks.max(axis=2), 0)"),
    ("block scale without s_g", "scale = (e4m3_decode(sf).astype(np.float32) * s_g).astype(np.float32)", "scale = e4m3_decode(sf).astype(np.float32)"),
    ("saturation count >=", "n_sat = int(np.count_nonzero(t > np.float32(E4M3_MAX)))", "n_sat = int(np.count_nonzero(t >= np.float32(E4M3_MAX)))"),
    ("element by division not reciprocal", "q = (blocks * r_s[:, :, None]).astype(np.float32)", "q = np.where(scale[:, :, None] == 0, np.float32(0) * blocks, blocks / np.where(scale == 0, np.float32(1), scale)[:, :, None]).astype(np.float32)"),
    ("ties to odd", "pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))", "pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 1))"),
    ("ties up", "pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))", "pick_hi = (d_hi <= d_lo)"),
    ("E2M1 sign dropped", "return code | (np.signbit(q).astype(np.uint8) << 3)", "return code"),
    ("nibbles swapped", "return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)", "return (c[:, 1::2] | (c[:, 0::2] << 4)).astype(np.uint8)"),
    ("scale layout lane/column swapped", "return (atom * 512 + (rows % 32) * 16 + ((rows % 128) // 32) * 4 + cols % 4).astype(np.int64)", "return (atom * 512 + (rows % 32) * 4 + ((rows % 128) // 32) * 128 + cols % 4).astype(np.int64)"),
    ("lambda without sqrt", "lam = np.where(ok, np.sqrt(ratio).astype(np.float32), np.float32(1.0)).astype(np.float32)", "lam = np.where(ok, ratio, np.float32(1.0)).astype(np.float32)"),
    ("lambda inverted", "ratio = np.where(ok, ax / np.where(ok, aw, np.float32(1)), np.float32(1)).astype(np.float32)", "ratio = np.where(ok, aw / np.where(ok, ax, np.float32(1)), np.float32(1)).astype(np.float32)"),
    ("s_g over 448 only", "s_g = np.float32(top / np.float32(E2M1_MAX * E4M3_MAX)) if top > 0 else np.float32(1.0)\n    return dict(ax=ax", "s_g = np.float32(top / np.float32(E4M3_MAX)) if top > 0 else np.float32(1.0)\n    return dict(ax=ax"),
    ("s_g from unsmoothed absmax", "smoothed = (ax * inv_lam).astype(np.float32)", "smoothed = ax.astype(np.float32)"),
    ("residual adds the branch", "r64 = w * lam[None, :] - lam[None, :] * acc", "r64 = w * lam[None, :] + lam[None, :] * acc"),
    ("residual branch without lambda", "r64 = w * lam[None, :] - lam[None, :] * acc", "r64 = w * lam[None, :] - acc"),
    ("down folds lambda the wrong way", "down = f64_to_bf16((l1 / lam[:, None]).T)", "down = f64_to_bf16((l1 * lam[:, None]).T)"),
    ("factor split uneven", "l1 = u[:, :rank] * root[None, :]", "l1 = u[:, :rank] * (root * root)[None, :]"),
    ("linear without weight tensor scale", "y = (np.float64(np.float32(s_g_act)) * np.float64(np.float32(s_g_w))) * (a @ w.T)", "y = np.float64(np.float32(s_g_act)) * (a @ w.T)"),
    ("linear subtracts the branch", "y = y + d @ bf16_to_f64(up_bits).T", "y = y - d @ bf16_to_f64(up_bits).T"),
    ("linear drops bias", "        y = y + bf16_to_f64(bias_bits)[None, :]\n    return y\n\n\ndef reference_linear", "        pass\n    return y\n\n\ndef reference_linear"),
    ("score without sqrt", "rel.append(math.sqrt(n_s / d_s) if d_s > 0", "rel.append((n_s / d_s) if d_s > 0"),
    ("score normalised by Yq", "d_s = float(np.sum(yr[b:e] * yr[b:e]))", "d_s = float(np.sum(yq[b:e] * yq[b:e]))"),
    ("bits lost in nats", "out[c, m] = float(np.mean(np.log2(ratio)))", "out[c, m] = float(np.mean(np.log(ratio)))"),
    ("bits lost over groups of 32", "group = np.repeat(chan.reshape(-1, BLOCK).max(axis=1), BLOCK)", "group = np.repeat(chan.reshape(-1, 2 * BLOCK).max(axis=1), 2 * BLOCK) if chan.size % 32 == 0 else np.repeat(chan.reshape(-1, BLOCK).max(axis=1), BLOCK)"),
    ("bits lost counts zero channels", "counted = chan > 0", "counted = chan >= 0"),
    ("grid exponent of aw wrong", "t = a64 * lx - (1.0 - a64) * lw", "t = a64 * lx - a64 * lw"),
    ("grid s_g with lambda", "top = np.float32((ax * inv).astype(np.float32).max()) if ax.size else np.float32(0)", "top = np.float32((ax * lam).astype(np.float32).max()) if ax.size else np.float32(0)"),
    ("selection by argmax", "return int(np.argmin(total))", "return int(np.argmax(total))"),
    ("alpha grid bounds", "def alpha_grid(n: int = 39, lo: float = 0.05, hi: float = 0.95)", "def alpha_grid(n: int = 39, lo: float = 0.0, hi: float = 1.0)"),
    ("MX exponent off by one", "e = np.where(amax > 0, e2.astype(np.int64) - 1 - E4M3_EMAX, -127)", "e = np.where(amax > 0, e2.astype(np.int64) - E4M3_EMAX, -127)"),
    ("MX scales multiply", "scaled = blocks * np.exp2(-e.astype(np.float64))[:, :, None]", "scaled = blocks * np.exp2(e.astype(np.float64))[:, :, None]"),
    ("MX bias 128", "return (vals * np.exp2(np.asarray(scales, np.float64) - 127.0)[:, :, None]).reshape(r, k)", "return (vals * np.exp2(np.asarray(scales, np.float64) - 128.0)[:, :, None]).reshape(r, k)"),
    ("MX zero block exponent 0", "e = np.where(amax > 0, e2.astype(np.int64) - 1 - E4M3_EMAX, -127)", "e = np.where(amax > 0, e2.astype(np.int64) - 1 - E4M3_EMAX, 0)"),
    ("E4M3 sign dropped", "    mag = E4M3_VALUES[b & 0x7F]\n    return np.where(b & 0x80, -mag, mag)", "    mag = E4M3_VALUES[b & 0x7F]\n    return mag"),
    ("reference linear drops bias", "    y = bf16_to_f64(x_bits) @ bf16_to_f64(w_bits).T\n    if bias_bits is not None:\n        y = y + bf16_to_f64(bias_bits)[None, :]", "    y = bf16_to_f64(x_bits) @ bf16_to_f64(w_bits).T\n    if bias_bits is not None:\n        pass"),
    ("weight tensor scale doubled", "cw = calib(r, None, None)", "cw = dict(s_g=np.float32(calib(r, None, None)['s_g'] * 2))"),
    ("score segment end inclusive", "diff = yq[b:e] - yr[b:e]", "diff = yq[b:e + 1] - yr[b:e + 1]"),
    ("row selection end inclusive", "idx = [np.arange(b, e) for b, e in segments]", "idx = [np.arange(b, min(e + 1, m)) for b, e in segments]"),
    ("bf16 decode shift", "(np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16)", "(np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 15)"),
    ("scale atoms overlap", "return (atom * 512 + (rows % 32) * 16", "return (atom * 256 + (rows % 32) * 16"),
    ("layer drops the low-rank branch", "d = lowrank_down(x_bits, down_bits) if down_bits is not None and down_bits.shape[0] else None", "d = None"),
    ("E4M3 no saturation", "code = _nearest_index_ties_even(np.minimum(t, E4M3_MAX), E4M3_VALUES)", "code = _nearest_index_ties_even(t, E4M3_VALUES[:-1])"),
]



def run_one(src: str, old: str, new: str):
    """Run the pins against the oracle with `old` replaced by `new`; returns (caught, first failure)."""
    assert src.count(old) == 1, old
    work = tempfile.mkdtemp(prefix="oracle_mutant_")
    try:
        os.makedirs(os.path.join(work, "oracle"))
        os.makedirs(os.path.join(work, "tests"))
        open(os.path.join(work, "oracle", "__init__.py"), "w").close()
        with open(os.path.join(work, "oracle", "svdq_oracle.py"), "w") as f:
            f.write(src.replace(old, new))
        for name in os.listdir(os.path.join(REPO, "tests")):
            if name.startswith("test_oracle") or name == "conftest.py":
                shutil.copy(os.path.join(REPO, "tests", name), os.path.join(work, "tests", name))
        shutil.copytree(os.path.join(REPO, "tests", "golden"), os.path.join(work, "tests", "golden"))
        shutil.copy(os.path.join(REPO, "synthetic.py"), os.path.join(work, "synthetic.py"))
        r = subprocess.run([sys.executable, "-m", "pytest", "tests", "-q", "-x", "-p", "no:cacheprovider"],
                           cwd=work, capture_output=True, text=True)
        failed = [l for l in r.stdout.splitlines() if l.startswith(("FAILED", "ERROR"))]
        return r.returncode != 0, (failed[0] if failed else "")
    finally:
        shutil.rmtree(work, ignore_errors=True)


def main() -> int:
    with open(SRC) as f:
        src = f.read()
    missed = 0
    for name, old, new in M:
        caught, first = run_one(src, old, new)
        missed += not caught
        print(f"{'caught' if caught else 'MISSED'}  {name}  {first}", flush=True)
    print(f"{len(M) - missed} of {len(M)} slips caught")
    return 1 if missed else 0


if __name__ == "__main__":
    sys.exit(main())

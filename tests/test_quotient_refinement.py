"""The rotate+quantize kernel forms y / s as a reciprocal product refined twice
with fused multiply-add residuals (Markstein's correction). This checks, in C on
the host with IEEE fp32 arithmetic (the same correctly rounded operations the
GPU executes), that the scheme returns exactly the IEEE quotient, including
dividends a few ulps from the half-integer points where the int8 code is
decided."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))


def test_refined_quotient_equals_ieee_division(tmp_path):
    exe = tmp_path / "quotient_check"
    subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-o", str(exe),
                           os.path.join(HERE, "csrc", "quotient_check.c"), "-lm"])
    out = subprocess.run([str(exe), "2000", "20000"], capture_output=True, text=True, check=True)
    bad, cases = map(int, out.stdout.split())
    assert cases == 40_000_000
    assert bad == 0, out.stderr


def test_division_by_127_in_one_correction_step(tmp_path):
    """The per-row scale s = max / 127 is formed as RN(max * RN(1/127)) plus one FMA
    correction; that equals the IEEE quotient for every positive finite float (a full
    sweep, about a minute, with H3Q_FULL_DIV127_SWEEP=1; by default every 61st bit
    pattern, which still covers every exponent and mantissa residue class mod 61)."""
    exe = tmp_path / "div127_check"
    subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-o", str(exe),
                           os.path.join(HERE, "csrc", "div127_check.c"), "-lm"])
    stride = "1" if os.environ.get("H3Q_FULL_DIV127_SWEEP") == "1" else "61"
    out = subprocess.run([str(exe), stride], capture_output=True, text=True, check=True)
    checked, wrong = map(int, out.stdout.split())
    assert checked >= 0x7F800000 // int(stride) - 1
    assert wrong == 0, out.stderr


def test_candidate_code_with_residual_check_equals_rounded_ieee_quotient(tmp_path):
    """The kernel's code decision: candidate rne(y rs) accepted when its residual
    |y - n s| is at most RN(s (1/2 - 2^-16)), else the refined quotient rounded half
    to even. Compared with rintf(y / s) on 40 M cases, a third of them exact
    half-integer quotients and a third within four ulps of one; the exact ties must
    all take the fallback."""
    exe = tmp_path / "code_check"
    subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-o", str(exe),
                           os.path.join(HERE, "csrc", "code_check.c"), "-lm"])
    out = subprocess.run([str(exe), "2000", "20000"], capture_output=True, text=True, check=True)
    bad, cases, fallbacks = map(int, out.stdout.split())
    assert cases == 40_000_000
    assert bad == 0, out.stderr
    assert fallbacks >= cases // 3


def test_code_check_catches_a_loose_residual_bound(tmp_path):
    """The same check with the bound at exactly s/2 (no margin for the rounding of y/s)
    must report mismatches: the exact half-integer quotients then pass the residual test
    with the wrong candidate."""
    exe = tmp_path / "code_check_loose"
    subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-DBOUND=0.5f", "-o", str(exe),
                           os.path.join(HERE, "csrc", "code_check.c"), "-lm"])
    out = subprocess.run([str(exe), "200", "2000"], capture_output=True, text=True, check=True)
    bad, cases, _ = map(int, out.stdout.split())
    assert cases == 400_000
    assert bad > 0

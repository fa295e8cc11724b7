"""The oracle's pins catch plausible mistakes.

Each case below plants one mistake in a copy of oracle/moe_oracle.c (a
dropped term, a flipped sign, a shifted index, a wrong constant, an
off-by-one range, another rounding rule), compiles the copy with the
oracle's own flags into a temporary library, and runs the CPU pin suites
against it through MOE_ORACLE_LIB.  Every mutant must fail at least one pin;
the unmodified copy, run the same way, must pass them all.  Nothing here
touches the GPU library.
"""
import concurrent.futures
import os
import shutil
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "moe_oracle.c")
PINS = ["tests/test_oracle_dispatch.py", "tests/test_oracle_combine.py",
        "tests/test_oracle_formats.py"]
CFLAGS = ["-O2", "-std=c11", "-fPIC", "-ffp-contract=off", "-fno-fast-math", "-shared"]

# name -> (text in the oracle, replacement)
MUTANTS = {
    "layout_tile_64": (
        "int32_t padded = (counts[e] + ORACLE_TILE - 1) / ORACLE_TILE * ORACLE_TILE;",
        "int32_t padded = (counts[e] + 63) / 64 * 64;"),
    "layout_rank_offset_shifted": (
        "rank_offsets[r] = offsets[r * El];",
        "rank_offsets[r] = offsets[r * El + 1];"),
    "layout_rank_count_drops_last_expert": (
        "for (int e = r * El; e < (r + 1) * El; ++e) s += counts[e];",
        "for (int e = r * El; e < (r + 1) * El - 1; ++e) s += counts[e];"),
    "layout_no_duplicate_check": (
        "if (ids[t * K + j] == e && status == OR_OK) status = OR_ERR_DUPLICATE_EXPERT;",
        "if (ids[t * K + j] == e + 100000 && status == OR_OK) status = OR_ERR_DUPLICATE_EXPERT;"),
    "layout_unstable_order": (
        "int32_t row = offsets[e] + fill[e]++;",
        "int32_t row = offsets[e] + (counts[e] - 1 - fill[e]++);"),
    "permute_first_padding_row_kept": (
        "for (int64_t p = (int64_t)offsets[e] + counts[e]; p < offsets[e + 1]; ++p)\n"
        "      memset(xp + p * row_bytes, 0, (size_t)row_bytes);",
        "for (int64_t p = (int64_t)offsets[e] + counts[e] + 1; p < offsets[e + 1]; ++p)\n"
        "      memset(xp + p * row_bytes, 0, (size_t)row_bytes);"),
    "combine_sign_flip": (
        "acc[h] += s * oracle_bf16_decode(yr[h]);",
        "acc[h] -= s * oracle_bf16_decode(yr[h]);"),
    "combine_drops_shared": (
        "for (int64_t h = 0; h < H; ++h) acc[h] += oracle_bf16_decode(shared[t * H + h]);",
        ";"),
    "combine_bwd_unscaled_grad_y": (
        "gy[h] = oracle_bf16_encode(s * gv);",
        "gy[h] = oracle_bf16_encode(gv);"),
    "combine_bwd_dot_index_shifted": (
        "dot += gv * oracle_bf16_decode(yr[h]);",
        "dot += gv * oracle_bf16_decode(yr[h ? h - 1 : 0]);"),
    "dispatch_bwd_wrong_row": (
        "const uint16_t* r = grad_xp + (int64_t)row * H;",
        "const uint16_t* r = grad_xp + (int64_t)(row ^ 1) * H;"),
    "quantize_447": (
        "float sc = amax > 0.0f ? amax / 448.0f : 1.0f;",
        "float sc = amax > 0.0f ? amax / 447.0f : 1.0f;"),
    "bf16_ties_away": (
        "double r = nearbyint(a / q) * q; /* a/q is exact: q is a power of two */",
        "double r = round(a / q) * q;"),
    "e4m3_subnormal_floor": (
        "if (ex < -6) ex = -6; /* subnormal spacing 2^-9 below 2^-6 */",
        "if (ex < -7) ex = -7;"),
    "tile_checksum_even_weights": (
        "acc += w * (2u * i + 1u);\n    }\n    if (xs) {",
        "acc += w * (2u * i);\n    }\n    if (xs) {"),
}


def _build(tmp, name, old, new):
    text = open(SRC).read()
    if old is not None:
        assert text.count(old) == 1, f"{name}: the text to mutate must occur exactly once"
        text = text.replace(old, new)
    d = os.path.join(tmp, name)
    os.makedirs(d)
    c = os.path.join(d, "moe_oracle.c")
    open(c, "w").write(text)
    lib = os.path.join(d, "libmoe_oracle.so")
    subprocess.run([shutil.which("gcc") or "gcc", *CFLAGS, "-o", lib, c, "-lm"], check=True,
                   capture_output=True)
    return lib


def _run_pins(lib):
    env = dict(os.environ, MOE_ORACLE_LIB=lib)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        "-m", "not gpu", *PINS], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=600)
    return r.returncode, (r.stdout + r.stderr)[-600:]


def test_every_mutant_fails_a_pin_and_the_original_passes(tmp_path):
    cases = [("original", None, None)] + [(n, o, m) for n, (o, m) in MUTANTS.items()]
    libs = {n: _build(str(tmp_path), n, o, m) for n, o, m in cases}
    with concurrent.futures.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 2)) as ex:
        results = dict(zip(libs, ex.map(_run_pins, libs.values())))
    rc, tail = results.pop("original")
    assert rc == 0, f"the unmodified oracle copy fails its pins:\n{tail}"
    survivors = [n for n, (rc, _) in results.items() if rc == 0]
    assert not survivors, f"mutants that pass every pin: {survivors}"
    for n, (rc, tail) in results.items():
        assert rc == 1, f"{n}: pytest did not report a test failure (rc={rc}):\n{tail}"

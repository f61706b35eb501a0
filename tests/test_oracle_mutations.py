"""Each plausible mistake planted in a copy of the oracle fails a pin.

The copy is built in a temporary directory on the CPU; the real oracle is
never modified.  Every mutation below must make ``test_oracle_pins.py`` fail,
which shows the pins constrain the gather index, the slice strides of A, B and
the rank activations, the column offset of B, the scaling, the K range, the
output row of each op and the orientation of B, and, for the base projection
with the expand folded in, the column offset of W, its gather row and its
scaling.
"""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTATIONS = {
    "gather_without_permutation": (
        "const uint16_t* xrow = x + (int64_t)permutation[i] * ld_x;",
        "const uint16_t* xrow = x + (int64_t)i * ld_x;"),
    "slice_stride_r_not_rs": (
        "const int64_t n = (int64_t)q * rs + j;",
        "const int64_t n = (int64_t)q * r + j;"),
    "B_without_column_offset": (
        "const uint16_t* brow = B + (c - slice_offsets[0]) * rs;",
        "const uint16_t* brow = B + (c) * rs;"),
    "scaling_dropped": ("float prod = scaling * acc;", "float prod = acc;"),
    "rank_block_stride_r": (
        "(const uint16_t*)in_r + (int64_t)i * ld_in + (int64_t)q * rs;",
        "(const uint16_t*)in_r + (int64_t)i * ld_in + (int64_t)q * r;"),
    "last_k_term_dropped": (
        "for (int k = 0; k < K; ++k)\n              acc += oracle_decode",
        "for (int k = 0; k < K - 1; ++k)\n              acc += oracle_decode"),
    "shrink_row_is_token": (
        "((uint16_t*)out_r)[(int64_t)i * ld_out + n]",
        "((uint16_t*)out_r)[(int64_t)permutation[i] * ld_out + n]"),
    "expand_row_is_sorted_row": (
        "uint16_t* o = (uint16_t*)base_out + t * ld_base + c;",
        "uint16_t* o = (uint16_t*)base_out + i * ld_base + c;"),
    "base_W_without_column_offset": (
        "const uint16_t* wrow = W + (c - slice_offsets[0]) * ld_w;",
        "const uint16_t* wrow = W + c * ld_w;"),
    "base_row_is_sorted_row": (
        "const uint16_t* xrow = x + t * ld_x;",
        "const uint16_t* xrow = x + (int64_t)i * ld_x;"),
    "base_scaling_dropped": (
        "const float sum = scaling == 0.0f ? base : base + scaling * lora;",
        "const float sum = scaling == 0.0f ? base : base + lora;"),
    "B_transposed": (
        "acc += oracle_decode(v[j], dtype) * oracle_decode(brow[j], dtype);",
        "acc += oracle_decode(v[j], dtype) * "
        "oracle_decode(B[(int64_t)j * n_tot + (c - slice_offsets[0])], dtype);"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_fails_a_pin(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(os.path.join(ROOT, "oracle", "lora_oracle.c")).read()
    assert src.count(old) == 1, "mutation anchor not found; update the mutation list"
    work = tmp_path / "copy"
    ign = shutil.ignore_patterns("*.so", "__pycache__")
    shutil.copytree(os.path.join(ROOT, "oracle"), work / "oracle", ignore=ign)
    (work / "scatter_gemm_b200").mkdir()
    shutil.copy(os.path.join(ROOT, "scatter_gemm_b200", "workloads.py"),
                work / "scatter_gemm_b200" / "workloads.py")
    (work / "scatter_gemm_b200" / "__init__.py").write_text("")
    (work / "tests").mkdir()
    for f in ("conftest.py", "test_oracle_pins.py"):
        shutil.copy(os.path.join(ROOT, "tests", f), work / "tests" / f)
    (work / "oracle" / "lora_oracle.c").write_text(src.replace(old, new))
    subprocess.check_call([sys.executable, str(work / "oracle" / "build.py"), "--force"],
                          stdout=subprocess.DEVNULL)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        str(work / "tests" / "test_oracle_pins.py")],
                       cwd=str(work), capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"mutation {name} passed every pin:\n{r.stdout[-2000:]}"

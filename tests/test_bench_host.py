"""Host-side helpers of bench.py (no GPU): the source hash that keys the DRAM
traffic records in profiles/traffic.txt ignores comments and blank lines and
nothing else (a record taken on other code must not be reported)."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

CODE = """// header
#include "x.h"
/* block
   comment */
__global__ void k(float *a) {   // trailing
    a[0] = 1.f;

}
"""


def test_code_only_drops_comments_and_blank_lines():
    assert bench.code_only(CODE) == '#include "x.h"\n__global__ void k(float *a) {\n    a[0] = 1.f;\n}'


def test_comment_edit_keeps_code_and_code_edit_changes_it():
    commented = CODE.replace("// trailing", "// reworded").replace("// header", "// other\n\n")
    assert bench.code_only(commented) == bench.code_only(CODE)
    assert bench.code_only(CODE.replace("1.f", "2.f")) != bench.code_only(CODE)



def test_e2e_step_count():
    # about 6 s of device time, 4 to 64 steps
    assert bench.e2e_step_count(351.4) == 17
    assert bench.e2e_step_count(1.6) == 64
    assert bench.e2e_step_count(3000.0) == 4
    assert bench.e2e_step_count(0.0) == 64

"""The in-tree build: every CUDA/C++ source and header of the library takes part
in the staleness check, so editing any of them rebuilds the library."""
from pathlib import Path

from expert_warp_top_b200 import build


def test_staleness_check_covers_every_source_and_header():
    csrc = Path(build.__file__).parent / "csrc"
    on_disk = {p for p in csrc.iterdir() if p.suffix in (".cu", ".cuh", ".h")}
    tracked = set(build.sources())
    assert on_disk and on_disk <= tracked
    assert any(p.name == "moe_occult.h" for p in tracked)

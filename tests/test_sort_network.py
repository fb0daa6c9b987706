"""The routing kernel's 8-input sorting network (csrc/route.cuh, kNet) sorts every input:
by the 0-1 principle it is enough that it sorts all 256 sequences of zeros and ones."""
import itertools
import re
from pathlib import Path

SRC = Path(__file__).resolve().parent.parent / "expert_warp_top_b200" / "csrc" / "route.cuh"


def network():
    text = SRC.read_text()
    m = re.search(r"kNet\[19\]\[2\] = \{(.*?)\};", text, re.S)
    assert m, "kNet not found"
    pairs = [(int(a), int(b)) for a, b in re.findall(r"\{(\d+), (\d+)\}", m.group(1))]
    assert len(pairs) == 19
    return pairs


def test_network_sorts_all_zero_one_inputs():
    net = network()
    assert all(0 <= i < j < 8 for i, j in net)
    for bits in itertools.product((0, 1), repeat=8):
        a = list(bits)
        for i, j in net:
            if a[i] > a[j]:
                a[i], a[j] = a[j], a[i]
        assert a == sorted(a), bits

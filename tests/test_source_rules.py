"""Static checks of the CUDA sources for the library's failure-reporting rules (no GPU needed):

* every spin on an mbarrier is bounded: a `while` that polls `mbar_try_wait` also reads the global
  timer (and gives up), and an unconditional loop reads the timer within its first lines;
* no kernel stops the device on purpose: no trap instruction and no device-side assert (errors go
  to the workspace's status block instead).
"""
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "parameter_space_moe_swimba_b200", "csrc")


def sources():
    for f in sorted(os.listdir(CSRC)):
        if f.endswith((".cu", ".cuh")):
            with open(os.path.join(CSRC, f)) as fh:
                yield f, fh.read().splitlines()


def test_every_mbarrier_spin_is_bounded_by_the_timer():
    checked = 0
    for name, lines in sources():
        for i, line in enumerate(lines):
            code = line.split("//")[0]
            window = "\n".join(l.split("//")[0] for l in lines[i:i + 6])
            if "while" in code and "mbar_try_wait(" in code:
                checked += 1
                assert "globaltimer_ns()" in window, f"{name}:{i + 1}: unbounded mbarrier spin"
            if re.search(r"while\s*\(\s*true\s*\)|for\s*\(\s*;\s*;\s*\)", code):
                checked += 1
                assert "globaltimer_ns()" in window and ("return" in window or "break" in window), (
                    f"{name}:{i + 1}: unconditional loop without a time limit")
    assert checked >= 5  # the pipelines' drains, the bounded wait itself, the on-purpose timeout


def test_no_trap_and_no_device_assert():
    for name, lines in sources():
        for i, line in enumerate(lines):
            code = line.split("//")[0]
            assert "__trap" not in code and not re.search(r"\btrap\s*;", code), f"{name}:{i + 1}"
            assert not re.search(r"(?<!static_)\bassert\s*\(", code), f"{name}:{i + 1}: device assert"

"""The committed ncu summaries describe the kernels as they are committed.

Each summary under profiles/ records the sha256 (first 16 hex digits) of the
kernel sources it was captured on and names those sources; a summary whose
digest no longer matches describes an earlier revision of its kernel and must
be recaptured.  Every ncu command in a summary leaves the GPU clocks alone
(`--clock-control none`).  No GPU needed.
"""
import hashlib
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PROFILES = os.path.join(ROOT, "profiles")
CSRC = os.path.join(ROOT, "bit_nf4_quantized_qlora_b200", "csrc")

SUMMARIES = sorted(f for f in os.listdir(PROFILES) if f.endswith(".txt"))


def _digest(names):
    h = hashlib.sha256()
    for name in names:
        with open(os.path.join(CSRC, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def test_there_are_summaries():
    assert len(SUMMARIES) >= 10


@pytest.mark.parametrize("name", SUMMARIES)
def test_summary_matches_the_committed_sources(name):
    text = open(os.path.join(PROFILES, name)).read()
    recorded = re.search(r"^kernel_source_sha256: (\w+)$", text, re.M)
    sources = re.search(r"^kernel_sources: (.+)$", text, re.M)
    assert recorded and sources, f"{name} names neither its digest nor its sources"
    names = sources.group(1).split()
    assert all(os.path.exists(os.path.join(CSRC, n)) for n in names), names
    assert _digest(names) == recorded.group(1), f"{name} was captured on other sources: recapture it"


@pytest.mark.parametrize("name", sorted(os.listdir(PROFILES)))
def test_every_ncu_command_leaves_the_clocks_alone(name):
    text = open(os.path.join(PROFILES, name)).read()
    for line in text.splitlines():
        if line.lstrip().startswith("ncu "):
            assert "--clock-control none" in line, f"{name}: {line.strip()}"

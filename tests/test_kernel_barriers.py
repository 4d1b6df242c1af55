"""Source check of the attention kernels' mbarrier sets (CPU).

Every kernel that synchronises its warp roles through shared-memory
mbarriers keeps them in one struct (``struct Bars...``). A barrier that is
waited on or arrived at without ``mbarrier.init`` makes the kernel read an
undefined phase, so every member of each such struct must be initialised by
an ``mbar_init(&bars.<member>...)`` in the same file, and no
``bars.<name>`` may name a barrier that the struct does not declare.
"""
import glob
import os
import re

import pytest

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "bit_attention_diffusion_b200", "csrc")
SOURCES = sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _strip_comments(src: str) -> str:
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return re.sub(r"//[^\n]*", "", src)


def _bar_structs(src: str):
    """{struct name: [member names]} for the structs of uint64_t barriers."""
    out = {}
    for m in re.finditer(r"struct\s+(Bars\w*)\s*\{(.*?)\};", src, flags=re.S):
        members = []
        for decl in re.finditer(r"uint64_t\s+([^;]+);", m.group(2)):
            for item in decl.group(1).split(","):
                name = re.match(r"\s*(\w+)", item)
                if name:
                    members.append(name.group(1))
        out[m.group(1)] = members
    return out


@pytest.mark.parametrize("path", SOURCES, ids=[os.path.basename(p) for p in SOURCES])
def test_every_barrier_is_initialised(path):
    src = _strip_comments(open(path).read())
    structs = _bar_structs(src)
    if not structs:
        pytest.skip("no barrier struct in this file")
    inited = set(re.findall(r"mbar_init\(\s*&bars\.(\w+)", src))
    used = set(re.findall(r"\bbars\.(\w+)", src))
    declared = {m for members in structs.values() for m in members}
    missing = declared - inited
    assert not missing, f"{os.path.basename(path)}: barriers never initialised: {sorted(missing)}"
    unknown = used - declared
    assert not unknown, f"{os.path.basename(path)}: bars.<name> not declared: {sorted(unknown)}"


def test_the_check_sees_the_attention_kernels():
    names = {os.path.basename(p) for p in SOURCES
             if _bar_structs(_strip_comments(open(p).read()))}
    assert {"attn_fp8.cu", "attn_fp4.cu", "attn_bf16.cu"} <= names


def test_the_check_catches_a_missing_init():
    src = ("struct Bars { uint64_t q, kfull[3], epi[2]; };\n"
           "void f() { mbar_init(&bars.q, 1); for (;;) mbar_init(&bars.kfull[i], 1);\n"
           "  // mbar_init(&bars.epi[i], 4);\n  wait(&bars.epi[0]); }")
    s = _strip_comments(src)
    inited = set(re.findall(r"mbar_init\(\s*&bars\.(\w+)", s))
    assert set(_bar_structs(s)["Bars"]) - inited == {"epi"}

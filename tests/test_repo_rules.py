"""Source hygiene, checked on the CPU: no source file, test, golden fixture
or build script names the project's planning documents or the tooling
around it, points at paths of a particular machine, quotes no stream-batch
copy call, and no kernel source issues a load with cluster multicast (the
library's peer transport must stay on plain loads and stores)."""
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
THIS = os.path.relpath(os.path.abspath(__file__), ROOT)

# each pattern is assembled from pieces so that this file does not match itself
FORBIDDEN = [
    ("planning documents", r"\b(" + "|".join(["BASE" + "LINE\\.(json|md)", "SUR" + "VEY",
                                               "VER" + "DICT", "AD" + "VICE\\.md",
                                               "DES" + "IGN\\.md", "REA" + "DME",
                                               "PA" + "PER\\.md", "north" + "_star"]) + r")"),
    ("machine paths", r"/" + r"root/"),
    ("remote GPU tool", r"\bgpu" + r"run\b"),
    ("batched copies", r"Memcpy" + r"(3D)?Batch"),
    ("cluster multicast", r"multicast::" + r"cluster"),
]


def _sources():
    out = subprocess.run(["git", "ls-files"], cwd=ROOT, capture_output=True, text=True)
    if out.returncode != 0:
        pytest.skip("not a git checkout")
    for f in out.stdout.split():
        if f == THIS or not re.search(r"\.(py|cu|cuh|h|c|cpp|sh|txt|toml|cfg)$", f):
            continue
        yield f


@pytest.mark.parametrize("what,pattern", FORBIDDEN, ids=[w for w, _ in FORBIDDEN])
def test_sources_do_not_name(what, pattern):
    rx = re.compile(pattern)
    hits = []
    for f in _sources():
        with open(os.path.join(ROOT, f), errors="replace") as fh:
            for n, line in enumerate(fh, 1):
                if rx.search(line):
                    hits.append("%s:%d: %s" % (f, n, line.strip()[:100]))
    assert not hits, "%s named in:\n%s" % (what, "\n".join(hits[:20]))

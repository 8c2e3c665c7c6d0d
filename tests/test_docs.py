"""The documents name files that exist: every `path` in backticks in the design doc,
README.md and the benchmark spec that looks like a source, header, test or profile
resolves to a file of the repository (relative to the root, the package or
its csrc/), and every command a profile summary quotes uses committed files."""
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PATTERN = re.compile(r"`([A-Za-z0-9_./-]+\.(?:cu|cuh|h|py|md|cpp|txt))`")


def _resolves(name):
    for base in ("", "rl_post_policy_b200", os.path.join("rl_post_policy_b200", "csrc")):
        if os.path.exists(os.path.join(ROOT, base, name)):
            return True
    return False


@pytest.mark.parametrize("doc", ["DESIGN.md", "README.md", "BASELINE.md"])
def test_named_files_exist(doc):
    text = open(os.path.join(ROOT, doc)).read()
    missing = sorted({m for m in PATTERN.findall(text) if not _resolves(m)})
    assert not missing, missing


def test_profile_commands_use_committed_files():
    prof = os.path.join(ROOT, "profiles")
    for name in os.listdir(prof):
        text = open(os.path.join(prof, name)).read()
        assert "_work/" not in text, name           # scratch files are not part of the product
        for script in re.findall(r"python ([A-Za-z0-9_./-]+\.py)", text):
            assert os.path.exists(os.path.join(ROOT, script)), (name, script)

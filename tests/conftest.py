import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size workloads (minutes of CPU oracle time)")


def read_golden(name):
    """Parse a golden fixture: '#' comments; '[section]' headers; rows of tokens."""
    sections, cur = {}, None
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            if line.startswith("[") and line.endswith("]"):
                cur = line[1:-1]
                sections[cur] = []
                continue
            sections.setdefault(cur, []).append(line.split())
    return sections


@pytest.fixture
def golden():
    return read_golden


def pytest_sessionstart(session):
    # A planted oracle mistake for the mutation check (tests/oracle_mutations.py);
    # unset in every ordinary run.
    name = os.environ.get("FFN_ORACLE_MUTATION")
    if name:
        import oracle_mutations
        oracle_mutations.apply(name)

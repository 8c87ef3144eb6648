import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the CUDA library")


# A planted oracle mistake for tests/test_oracle_mutations.py (which runs the oracle's pins in
# a child pytest process with this variable set); unset in every normal run.
_MUTANT = os.environ.get("AWQ_ORACLE_MUTANT")
if _MUTANT:
    sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
    import oracle_mutants  # noqa: E402

    oracle_mutants.install(_MUTANT)

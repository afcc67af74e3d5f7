import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def src():
    import dckv_synth

    return dckv_synth.source(0)


@pytest.fixture(scope="session")
def codec_literal(src):
    import dckv_synth

    return dckv_synth.codec(src, step_scale=1.0, literal_b=True)


@pytest.fixture(scope="session")
def codec_55(src):
    """The ~220 B/token codec of the single 4,096-token configuration (calibrated step scale)."""
    import dckv_synth

    return dckv_synth.calibrated_codec(src, 220.0, 16)


@pytest.fixture(scope="session")
def codec_centred(src):
    """Mean models scaled up so that centres are non-zero in both passes."""
    import dckv_synth

    return dckv_synth.codec(src, step_scale=None, target_bytes=220.0, embed_std=1.0,
                            mean_gain=1.0, neigh_gain=40.0)


def golden(name):
    import json

    with open(os.path.join(ROOT, "tests", "golden", name)) as f:
        return json.load(f)

"""Shared pytest set-up: repository root on sys.path and the ``gpu`` marker.

Tests marked ``gpu`` need a CUDA device and the built CUDA library; all
others run on the CPU.
"""

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
HERE = os.path.dirname(os.path.abspath(__file__))
if HERE not in sys.path:
    sys.path.insert(0, HERE)


def pytest_configure(config):
    config.addinivalue_line(
        "markers", "gpu: needs a CUDA device and the built CUDA library")

"""Shared pytest configuration.

Markers:
  gpu -- needs a B200 (sm_100a) and the built CUDA library; run with -m gpu.
Everything unmarked runs on a CPU-only machine.
"""
from __future__ import annotations

import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 GPU and the built CUDA library")
    # build (if stale) the oracle and the CUDA library before test modules import them
    # (the package's build script is loaded by path: importing the package
    # itself requires the built library)
    import importlib.util
    from oracle import build as oracle_build
    oracle_build.build()
    spec = importlib.util.spec_from_file_location(
        "_eqlin_build", os.path.join(ROOT, "cyclic_group_dft_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()


@pytest.fixture(scope="session")
def golden_dir() -> str:
    return os.path.join(ROOT, "tests", "golden")


def parse_blocks(path: str) -> list[dict]:
    """Parse a golden file of 'key values...' lines grouped by 'name'/'end'."""
    blocks, cur = [], None
    with open(path) as f:
        for raw in f:
            line = raw.split("#", 1)[0].strip()
            if not line:
                continue
            key, *vals = line.split()
            if key == "name":
                cur = {"name": vals[0]}
            elif key == "end":
                blocks.append(cur)
                cur = None
            else:
                cur[key] = [float(v) for v in vals]
    return blocks


def parse_facts(path: str) -> dict:
    facts = {}
    with open(path) as f:
        for raw in f:
            line = raw.split("#", 1)[0].strip()
            if line:
                key, *vals = line.split()
                facts[key] = [float(v) for v in vals]
    return facts

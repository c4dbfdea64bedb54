"""Source rules of the CUDA path, checked on the host.

* No bulk or tensor copy with cluster multicast: every TMA / bulk load of the
  library reads into its own CTA (the CTA pair shares work through
  cta_group::2 MMAs and commit arrivals, which may multicast), so that no
  path, on any number of GPUs, issues a multicast load.
* None of the batched copy entry points of the runtime or driver API (the
  library issues its own kernels and single copies only).
* Every asynchronous copy instruction in the sources is one of the known
  forms, so that a new one is looked at before it lands."""
import os
import re

import pytest

CSRC = os.path.join(os.path.dirname(__file__), "..", "w8a8_quantized_linear_b200", "csrc")
SOURCES = sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cu", ".cuh")))


def _text(path):
    with open(path, encoding="utf-8") as f:
        return f.read()


@pytest.mark.parametrize("path", SOURCES, ids=os.path.basename)
def test_no_multicast_copy(path):
    for line in _text(path).splitlines():
        if "cp.async.bulk" in line:
            assert "multicast" not in line, line.strip()


@pytest.mark.parametrize("path", SOURCES, ids=os.path.basename)
def test_no_batched_copy_calls(path):
    # the names are assembled here so that this file does not spell them
    names = [p + "Memcpy" + d + "Batch" + "Async" for p in ("cuda", "cu") for d in ("", "3D")]
    text = _text(path)
    for n in names:
        assert n not in text, n


KNOWN_COPY_FORMS = {
    "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes",
    "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes",
    "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes",
    "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group",
    "cp.async.bulk.commit_group",
    "cp.async.bulk.wait_group",
    "cp.async.bulk.wait_group.read",
}


def test_copy_forms_are_known():
    found = set()
    for path in SOURCES:
        for m in re.finditer(r"cp\.async\.bulk[\w.:]*", _text(path)):
            found.add(m.group(0).rstrip("."))
    assert found, "no copy instructions found"
    assert found <= KNOWN_COPY_FORMS, sorted(found - KNOWN_COPY_FORMS)

"""Host-side helpers of bench.py that need no GPU: the L2 read-flush buffer
and its label, and the whole-job throughput of independent replicas."""
import argparse

import pytest


def test_flush_buffer_size_and_label():
    import bench
    a = argparse.Namespace(flush_mib=256)
    f = bench._make_flush(a, "cpu")
    assert f.numel() * f.element_size() == 256 << 20
    assert bench._l2_note(a) == "flushed (256 MiB read) before each step, outside the step's event bracket"
    assert bench._l2_note(a, "once before each step") == "flushed (256 MiB read) once before each step"


def test_no_flush_is_labelled_a_diagnostic():
    import bench
    a = argparse.Namespace(flush_mib=0)
    assert bench._make_flush(a, "cpu").sum() is None
    assert "not a bench value" in bench._l2_note(a)


def test_job_throughput_of_replicas():
    import bench
    # two replicas, 2.61e11 operations each, the slower one taking 65 us
    assert bench._job_tops(2.61e11, 0.065, 2) == pytest.approx(2 * 2.61e11 / 65e-6 / 1e12)

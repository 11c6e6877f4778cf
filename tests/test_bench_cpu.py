"""Host-side checks of bench.py's bookkeeping (no GPU): recorded DRAM traffic is
matched to kernel code, not to comments, every record in the committed
profile file is found for the current sources, and the side workloads timed
beside the main line are the ones their names say."""

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_code_hash_ignores_comments_and_whitespace(tmp_path):
    a = tmp_path / "a.cu"
    b = tmp_path / "b.cu"
    c = tmp_path / "c.cu"
    a.write_text("// header\nint f(int x) {\n  return x + 1;  // add one\n}\n/* block\n comment */\n")
    b.write_text("int f(int x) { return x + 1; }\n")
    c.write_text("int f(int x) { return x + 2; }\n")
    assert bench._sha(str(a)) == bench._sha(str(b))
    assert bench._sha(str(a)) != bench._sha(str(c))


def test_traffic_records_are_well_formed_and_looked_up_by_code_hash():
    sources = {"fa_bwd_tiles": bench.TILES_SOURCE, "fa_fwd": bench.FWD_SOURCE, "fa_decode": bench.DECODE_SOURCE}
    with open(bench.TRAFFIC_FILE) as f:
        records = [line.split() for line in f if line.strip() and not line.startswith("#")]
    assert records
    for kernel, workload, code_hash, nbytes in records:
        assert kernel in sources and int(nbytes) > 0 and len(code_hash) == 16
        got = bench._traffic(kernel, sources[kernel], workload)
        # the value is reported only while the kernel code is the one captured
        assert got == (float(nbytes) if bench._sha(sources[kernel]) == code_hash else None)
        # a record is tied to its workload
        assert bench._traffic(kernel, sources[kernel], workload + "_other") is None


def test_peaks_come_from_the_measured_file_when_present():
    peaks, src = bench._peaks()
    if os.path.exists(os.path.join(ROOT, "MEASURED_PEAKS.json")):
        assert src == "measured"
    assert peaks["hbm_gbs"] > 1000 and peaks["bf16_tflops"] > 500


def test_side_workloads_are_named_by_their_shapes():
    """The per-call timings beside the main line cover the other d = 128
    dropout workload and both wide head dims, each named by its shape."""
    from exact_io_aware_49_b200 import workloads as wl
    ws = [wl.BY_NAME[o] if isinstance(o, str) else o for o in bench.OTHER_WORKLOADS]
    for w in ws:
        assert w.name == f"causal_dropout_N{w.N}_d{w.d}", w.name
        assert w.causal and w.p_drop == 0.1 and w.backward
    assert sorted(w.d for w in ws) == [128, 192, 256]
    assert len({w.seed for w in ws}) == len(ws)

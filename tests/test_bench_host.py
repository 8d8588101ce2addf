"""Host-side parts of bench.py that need no GPU."""
import importlib.util
import json
from pathlib import Path

ROOT = Path(__file__).resolve().parents[1]


def _load_bench():
    spec = importlib.util.spec_from_file_location("bench_host_mod", ROOT / "bench.py")
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_traffic_record_is_for_the_current_kernel():
    """The bench line's roofline traffic comes from a committed ncu capture and
    is reported only while the search kernel's source is the one captured: the
    record must name the current source hash, so the figure is not stale."""
    bench = _load_bench()
    rec = json.loads((ROOT / "profiles" / "search_pair_kernel_traffic.json").read_text())
    assert rec["source_hash"] == bench.kernel_source_hash()
    t = bench.search_traffic("attn4096")
    assert t is not None and t == float(rec["per_launch_bytes"]["attn4096"])
    # algorithmic bytes of the workload: W and X once (fp16)
    assert t >= 2 * 4096 * 4096 * 2


def test_unknown_workload_has_no_traffic_figure():
    bench = _load_bench()
    assert bench.search_traffic("no_such_layer") is None

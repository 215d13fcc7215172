"""bench.py's traffic records (CPU only): kernel names from ncu's several
naming styles, the ingest of a raw-page CSV export, and the rule that a
record is used only while the kernel sources hash to the value it was taken
at."""
import csv
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_kernel_base_names():
    f = bench.kernel_base_name
    assert f("tc_state_kernel(CUtensorMap_st, CUtensorMap_st, TcStateParams)") == "tc_state_kernel"
    assert f("void tc_apply_kernel<0>(CUtensorMap_st, CUtensorMap_st, TcApplyParams)") == \
        "tc_apply_kernel"
    assert f("gla::combine_bulk_kernel(gla::CombineParams)") == "combine_bulk_kernel"
    assert f("void gla::tc_apply_kernel<0>(CUtensorMap_st, gla::TcApplyParams)") == \
        "tc_apply_kernel"
    assert f("void at::vectorized_elementwise_kernel<4, at::FillFunctor<float>, "
             "std::array<char *, 1>>(int, T2, T3)") == "vectorized_elementwise_kernel"


def _write_csv(path, rows):
    head = ["ID", "Kernel Name", "dram__bytes_read.sum", "dram__bytes_write.sum",
            "gpu__time_duration.sum"]
    units = ["", "", "Mbyte", "Kbyte", "us"]
    with open(path, "w", newline="") as fh:
        w = csv.writer(fh)
        w.writerow(head)
        w.writerow(units)
        for i, r in enumerate(rows):
            w.writerow([str(i), *r])


def test_ingest_means_and_hash(tmp_path, monkeypatch):
    traffic = tmp_path / "traffic.json"
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(traffic))
    src = tmp_path / "list.csv"
    _write_csv(src, [
        ("void gla::tc_apply_kernel<0>(CUtensorMap_st)", "400", "8", "90"),
        ("tc_apply_kernel(CUtensorMap_st)", "404", "12", "94"),
        ("tc_state_kernel(CUtensorMap_st)", "300", "0", "60"),
    ])
    bench.ingest_ncu(str(src), "720p")
    doc = json.loads(traffic.read_text())
    ap = doc["tc_apply_kernel"]["720p"]
    assert ap["launches"] == 2
    assert ap["bytes_per_launch"] == int(round((400e6 + 8e3 + 404e6 + 12e3) / 2))
    assert abs(ap["duration_us_under_ncu"] - 92.0) < 1e-9
    assert ap["source_sha"] == bench.source_sha()
    assert bench.traffic_for("tc_apply_kernel", "720p") == ap["bytes_per_launch"]
    assert bench.traffic_for("tc_apply_kernel", "480p") is None
    # a record taken on other sources is not used
    doc["tc_apply_kernel"]["720p"]["source_sha"] = "0" * 16
    traffic.write_text(json.dumps(doc))
    assert bench.traffic_for("tc_apply_kernel", "720p") is None


def test_committed_records_name_real_kernels():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as fh:
        doc = json.load(fh)
    names = set(doc) - {"_note"}
    assert {"tc_state_kernel", "tc_apply_kernel", "anchor_attn_kernel"} <= names
    for name in names:
        assert name.isidentifier(), name
        for rec in doc[name].values():
            assert rec["bytes_per_launch"] >= 0 and len(rec["source_sha"]) == 16

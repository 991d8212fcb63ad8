"""bench.py's measurement records, on a temporary tree (CPU only).

`--record-traffic` turns an ncu raw-page CSV into profiles/traffic.json (DRAM
read + write bytes per timed call, summed over the call's kernels, units
scaled); the bench line reports a recorded figure only while the sources it
was captured from hash the same, and null otherwise.  The committed records
are never touched: ROOT points at a copy."""
import csv
import json
import os

import pytest

import bench


def _tree(tmp_path):
    srcs = set(bench._TRAFFIC_COMMON) | set(bench._MASK_INST_SOURCES)
    for kernels, files in bench._TRAFFIC_CALLS.values():
        srcs |= set(files)
    for s in srcs:
        p = tmp_path / s
        p.parent.mkdir(parents=True, exist_ok=True)
        p.write_text(f"// source {s}\n")
    (tmp_path / "profiles").mkdir()
    return tmp_path


def _csv(path, rows):
    hdr = ["ID", "Kernel Name", "dram__bytes_read.sum", "dram__bytes_write.sum", "gpu__time_duration.sum"]
    units = ["", "", "Mbyte", "Kbyte", "us"]
    with open(path, "w", newline="") as fh:
        w = csv.writer(fh)
        w.writerow(hdr)
        w.writerow(units)
        for i, (name, rd, wr) in enumerate(rows):
            w.writerow([str(i), name, rd, wr, "1.0"])


FWD = "void bf16::attn_fwd_persist_kernel<64, 0>(CUtensorMap_st, CUtensorMap_st, CUtensorMap_st, bf16::FwdParams)"
DOT = "void bwd::dot_kernel<64>(const __nv_bfloat16 *, const __nv_bfloat16 *, gsa::TokLayout, long)"
DQ = "void bwd::dq_persist_kernel<0>(CUtensorMap_st, CUtensorMap_st, CUtensorMap_st, CUtensorMap_st, bwd::Params)"
DKV = "void bwd::dkdv_persist_kernel<0>(CUtensorMap_st, CUtensorMap_st, CUtensorMap_st, CUtensorMap_st, bwd::Params)"


def test_traffic_record_sums_scales_and_expires(tmp_path, monkeypatch):
    root = _tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(root))
    raw = root / "raw.csv"
    # the first launch of each kernel counts; the later one is ignored
    _csv(raw, [(FWD, "370.5", "84,000.0"), (DOT, "204.5", "7,695.1"), (DQ, "493.9", "86,446.0"),
               (DKV, "483.0", "171,934.4"), (FWD, "999.0", "1.0")])
    bench.record_traffic(str(raw), "ncu ... (test)")
    rec = json.load(open(root / "profiles" / "traffic.json"))
    assert rec["gsa_attn_fwd"]["bytes_per_launch"] == int(370.5e6 + 84000.0e3)
    bwd = rec["gsa_attn_bwd"]
    assert bwd["per_kernel"]["dq_persist_kernel<0>"] == int(493.9e6 + 86446.0e3)
    assert bwd["bytes_per_launch"] == sum(bwd["per_kernel"].values())
    assert set(bwd["per_kernel"]) == set(bench._TRAFFIC_CALLS["gsa_attn_bwd"][0])
    assert bwd["capture"] == "ncu ... (test)"
    # reported while the sources hash the same ...
    assert bench._traffic_record("gsa_attn_fwd") == rec["gsa_attn_fwd"]["bytes_per_launch"]
    assert bench._traffic_record("gsa_attn_bwd") == bwd["bytes_per_launch"]
    # ... and null after any of them changes (here a file only the backward lists)
    (root / bench._TRAFFIC_CALLS["gsa_attn_bwd"][1][-1]).write_text("// edited\n")
    assert bench._traffic_record("gsa_attn_bwd") is None
    assert bench._traffic_record("gsa_attn_fwd") == rec["gsa_attn_fwd"]["bytes_per_launch"]
    # a common source changes both
    (root / bench._TRAFFIC_COMMON[0]).write_text("// edited\n")
    assert bench._traffic_record("gsa_attn_fwd") is None


def test_call_missing_a_kernel_is_not_recorded(tmp_path, monkeypatch):
    root = _tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(root))
    raw = root / "raw.csv"
    _csv(raw, [(FWD, "1.0", "1.0"), (DOT, "1.0", "1.0"), (DQ, "1.0", "1.0")])   # no dK/dV launch
    bench.record_traffic(str(raw), "")
    rec = json.load(open(root / "profiles" / "traffic.json"))
    assert "gsa_attn_fwd" in rec and "gsa_attn_bwd" not in rec
    assert bench._traffic_record("gsa_attn_bwd") is None


def test_no_record_file_reads_as_null(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench._traffic_record("gsa_attn_fwd") is None
    assert bench._mask_inst_record() is None


def test_committed_records_name_existing_sources():
    # the committed records point at files of this tree (whether or not they still match)
    for name in ("traffic.json", "mask_inst.json"):
        rec = json.load(open(os.path.join(bench.ROOT, "profiles", name)))
        recs = rec.values() if name == "traffic.json" else [rec]
        for r in recs:
            for s in r["sources"]:
                assert os.path.exists(os.path.join(bench.ROOT, s)), s


class _FakeCsr:
    """The fields csr_nnz reads, on the CPU (no library needed)."""

    def __init__(self, row_ptr, w, classes):
        import torch
        self.row_ptr = torch.tensor(row_ptr, dtype=torch.int32)
        self.nblk = self.row_ptr.shape[2] - 1
        self.w, self.classes = w, classes

    def stored(self, c):
        return not (c == 0 and self.classes & 8)


def test_csr_nnz_counts_an_implicit_local_window():
    # two samples, 5 blocks, w = 2: the local window holds min(i, 2) + 1 blocks in row i
    # (1 + 2 + 3 + 3 + 3 = 12), the closed form N (w + 1) - w (w + 1) / 2 of the mask equation
    n, w = 5, 2
    rp = [[[0] * (n + 1), [0, 1, 2, 4, 5, 8], [0, 1, 3, 6, 9, 12]] for _ in range(2)]
    implicit = bench.csr_nnz(_FakeCsr(rp, w, 7 | 8))
    assert implicit[:, 0].tolist() == [n * (w + 1) - w * (w + 1) // 2] * 2 == [12, 12]
    assert implicit[:, 1].tolist() == [8, 8] and implicit[:, 2].tolist() == [12, 12]
    # stored lists count from their pointers
    rp[0][0] = [0, 1, 3, 6, 9, 12]
    rp[1][0] = [0, 1, 3, 6, 9, 12]
    assert bench.csr_nnz(_FakeCsr(rp, w, 7))[:, 0].tolist() == [12, 12]
    # a window wider than the sample: the whole causal triangle
    assert bench.csr_nnz(_FakeCsr(rp, 9, 1 | 8))[:, 0].tolist() == [15, 15]

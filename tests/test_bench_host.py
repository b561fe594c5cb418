"""Host-side logic of bench.py (no GPU): the packed copy layout of the
end-to-end leg, and the ncu traffic records behind the roofline's `traffic`."""
import json
import os
import sys

import numpy as np
import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def test_pack_offsets_are_aligned_and_disjoint():
    sizes = [128, 2097152, 8192, 1, 0, 300]
    offs, total = bench._pack_offsets(sizes)
    assert offs[0] == 0
    for (o, n), o_next in zip(zip(offs, sizes), offs[1:] + [total]):
        assert o % 256 == 0
        assert o + n <= o_next                    # no block runs into the next one
        assert o_next - o < n + 256 or n == 0     # padding below one alignment unit
    assert total % 256 == 0 and total >= sum(sizes)


def test_views_alias_their_block_of_the_packed_buffer():
    arrays = [np.arange(32, dtype=np.int32).reshape(32, 1),
              (np.arange(2 * 4 * 8, dtype=np.uint16) * 3).reshape(2, 1, 4, 8),
              np.arange(2 * 4 * 16, dtype=np.uint8).reshape(2, 1, 4, 16),
              np.linspace(-1, 1, 2 * 4, dtype=np.float32).reshape(2, 1, 4)]
    dtypes = [torch.int32, torch.bfloat16, torch.uint8, torch.float32]
    offs, total = bench._pack_offsets([a.nbytes for a in arrays])
    buf = torch.zeros(total, dtype=torch.uint8)
    for a, off in zip(arrays, offs):
        buf[off:off + a.nbytes] = torch.from_numpy(a.view(np.uint8).reshape(-1))
    for a, dt, off in zip(arrays, dtypes, offs):
        v = bench._view(buf, off, dt, a.shape, torch)
        assert tuple(v.shape) == a.shape and v.dtype == dt
        assert v.is_contiguous()
        got = v.contiguous().view(torch.uint8).numpy().reshape(-1)
        assert np.array_equal(got, a.view(np.uint8).reshape(-1))


def _write_ncu_csv(path, launches):
    """A capture in ncu's long CSV layout, with one of ncu's own log lines."""
    with open(path, "w") as f:
        f.write("==PROF== Connected to process 1\n")
        f.write('"ID","Kernel Name","Metric Name","Metric Unit","Metric Value"\n')
        for i, (name, rd, wr, us) in enumerate(launches):
            for m, u, v in (("dram__bytes_read.sum", "Mbyte", rd),
                            ("dram__bytes_write.sum", "Kbyte", wr),
                            ("gpu__time_duration.sum", "usecond", us)):
                f.write('"%d","%s","%s","%s","%s"\n' % (i, name, m, u, v))


def test_record_ncu_averages_matching_launches(tmp_path):
    csv_path = str(tmp_path / "cap.csv")
    out = str(tmp_path / "traffic.json")
    _write_ncu_csv(csv_path, [
        ("void index_score_tc_kernel<64, 1>(CUtensorMap_st)", "100.0", "400.0", "27.0"),
        ("void topk_reg_kernel<16, 4, 0, 0>(const float *)", "4.0", "0", "13.0"),
        ("void index_score_tc_kernel<64, 1>(CUtensorMap_st)", "102.0", "600.0", "29.0"),
    ])
    rec = bench.record_ncu(csv_path, "score", "decode_128k_full", "ncu ... (test)",
                           out_path=out)
    assert rec["launches"] == 2
    assert rec["dram_read_bytes_per_launch"] == 101.0e6
    assert rec["dram_write_bytes_per_launch"] == 500.0e3
    assert rec["dram_bytes_per_launch"] == 101.0e6 + 500.0e3
    assert rec["duration_us_under_ncu"] == 28.0
    assert rec["sources_sha1"] == bench.sources_sha1("score")
    # a second capture of the same kernel and workload replaces the first
    _write_ncu_csv(csv_path, [("void index_score_tc_kernel<64, 1>(x)", "90", "0", "20")])
    bench.record_ncu(csv_path, "score", "decode_128k_full", "again", out_path=out)
    caps = json.load(open(out))["captures"]
    assert len(caps) == 1 and caps[0]["dram_read_bytes_per_launch"] == 90e6


def test_profiled_traffic_lookup(tmp_path, monkeypatch):
    path = str(tmp_path / "traffic.json")
    sha = bench.sources_sha1("attn")
    doc = {"captures": [
        {"kernel": "attn", "sources_sha1": sha, "workload": "decode_128k_full",
         "dram_bytes_per_launch": 26.0e6},
        {"kernel": "attn", "sources_sha1": sha, "workload": "small_case",
         "dram_bytes_per_launch": 2.0e6, "units": 1000.0, "unit_kind": "selected"},
    ]}
    with open(path, "w") as f:
        json.dump(doc, f)
    monkeypatch.setattr(bench, "TRAFFIC_FILE", path)
    # the workload's own capture
    v, why = bench.profiled_traffic("attn", "decode_128k_full", 5.0)
    assert v == 26.0e6 and "this workload" in why
    # another workload: the capture with a unit count, scaled
    v, why = bench.profiled_traffic("attn", "other", 3000.0)
    assert v == 6.0e6 and "scaled" in why
    # no capture of the kernel's current sources at all
    monkeypatch.setattr(bench, "sources_sha1", lambda k: "0" * 40)
    v, why = bench.profiled_traffic("attn", "decode_128k_full", 5.0)
    assert v is None and "sources changed" in why


def test_profiled_traffic_without_a_unit_count(tmp_path, monkeypatch):
    path = str(tmp_path / "traffic.json")
    with open(path, "w") as f:
        json.dump({"captures": [{"kernel": "topk", "sources_sha1": bench.sources_sha1("topk"),
                                 "workload": "decode_128k_full",
                                 "dram_bytes_per_launch": 4.2e6}]}, f)
    monkeypatch.setattr(bench, "TRAFFIC_FILE", path)
    v, why = bench.profiled_traffic("topk", "prefill_chunk_4096_full", 1.0)
    assert v is None and "no ncu capture of this workload" in why

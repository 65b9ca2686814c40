"""Host arithmetic of bench.py, checked on the CPU: the roofline (which bound
sets it and the achieved fraction), the algorithmic work of each kernel at
the 78-layer stack's shape, the whole-job throughput of replicas, and the
rule that a recorded DRAM-traffic figure is reported only while the kernel
sources it was taken on are unchanged."""
import math

import pytest

import bench


def test_roofline_takes_the_slower_bound():
    hbm, tf = 6552.6, 1652.9
    # 6552.6 MB at the copy peak is 1 ms; 1 GFLOP at the tensor peak is ~0.6 us
    assert bench.roofline_time_us(6552.6e6, 1e9, hbm, tf) == pytest.approx(1000.0)
    assert bench.roofline_time_us(1.0, 1652.9e9, hbm, tf) == pytest.approx(1000.0)
    r = bench.roofline_of(6552.6e6, 1e9, 2000.0, hbm, tf)  # HBM-bound, timed at twice its roofline
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["achieved"] == pytest.approx(3276.3) and r["frac"] == pytest.approx(0.5)
    r = bench.roofline_of(1.0, 1652.9e9, 4000.0, hbm, tf)  # tensor-bound, four times its roofline
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["achieved"] == pytest.approx(413.225) and r["frac"] == pytest.approx(0.25)


def test_work_at_the_stack_shape():
    # indexer: 32 queries x 64 heads x 128 dims against 131072 shared bf16 keys
    by, fl = bench.indexer_work(32, 131072, 64, 128, 256, shared=True)
    assert fl == 2.0 * 32 * 64 * 128 * 131072  # 68.7 GFLOP
    assert by == 131072 * 256 + 32 * 64 * 128 * 2 + 32 * 64 * 4 + 32 * 131072 * 4
    # per-query caches read every key once per query
    by_pq, _ = bench.indexer_work(8, 131072, 64, 128, 256, shared=False)
    assert by_pq == 8 * 131072 * 256 + 8 * 64 * 128 * 2 + 8 * 64 * 4 + 8 * 131072 * 4
    # top-k: the score rows read, the index rows written
    assert bench.topk_work(32, 131072, 2048) == 32 * 131072 * 4 + 32 * 2048 * 4
    # sparse MLA: 2 B H k (576 + 512) FLOP, 18.25 GFLOP per layer
    _, fl = bench.mla_work(44613, 32, 128, 2048, gate=True)
    assert fl == pytest.approx(18.253611008e9)
    by_g, _ = bench.mla_work(1000, 32, 128, 2048, gate=True)
    by_n, _ = bench.mla_work(1000, 32, 128, 2048, gate=False)
    assert by_g - by_n == 32 * 128 * 512 * 2  # the gate logits, read once


def test_replica_throughput_and_cpu_baseline_formula():
    # 8 ranks x 32 queries x 20 steps over the slowest rank's 100 ms
    assert bench.replica_value(8, 32, 20, 100.0) == pytest.approx(8 * 32 * 20 / 0.1)
    # one decoded token: 21 F layers (indexer + top-k + attention) and 57 S
    # layers (attention only)
    tf, ta = 0.3, 0.05
    assert bench.cpu_tokens_per_s(tf, ta) == pytest.approx(1.0 / (21 * tf + 78 * ta))


def _write_launch_csv(path, rows):
    head = '"ID","Process ID","Kernel Name","Metric Name","Metric Unit","Metric Value"\n'
    body = "".join(f'"{i}","1","{k}","{m}","{u}","{v}"\n' for i, k, m, u, v in rows)
    path.write_text(head + body)


def test_traffic_figure_only_for_the_sources_it_was_taken_on(tmp_path, monkeypatch, capsys):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (tmp_path / "k.cu").write_text("kernel source, first version\n")
    prof = tmp_path / "profiles"
    prof.mkdir()
    csv = tmp_path / "dram.csv"
    # two launches of each of two kernels; the first launch of each counts
    _write_launch_csv(csv, [
        (0, "void main_kernel<256>(args)", "dram__bytes_read.sum", "byte", "1,000"),
        (0, "void main_kernel<256>(args)", "dram__bytes_write.sum", "byte", "200"),
        (1, "void combine_kernel(args)", "dram__bytes_read.sum", "byte", "30"),
        (1, "void combine_kernel(args)", "dram__bytes_write.sum", "byte", "0"),
        (2, "void main_kernel<256>(args)", "dram__bytes_read.sum", "byte", "9999"),
        (3, "void other_kernel(args)", "dram__bytes_read.sum", "byte", "5"),
    ])
    bench.ncu_traffic(str(csv), "kk", "main_kernel|combine_kernel", ["k.cu"])
    block = capsys.readouterr().out
    assert "traffic-dram-bytes-per-launch: 1230" in block
    (prof / "kk.md").write_text("# notes\n\n" + block)
    assert bench.load_traffic("kk") == 1230
    assert bench.load_traffic("another kernel") is None
    (tmp_path / "k.cu").write_text("kernel source, second version\n")
    assert bench.load_traffic("kk") is None  # taken on other sources: not reported


def test_launch_list_shares(tmp_path, capsys):
    csv = tmp_path / "launches.csv"
    _write_launch_csv(csv, [
        (0, "void a_kernel(x)", "gpu__time_duration.sum", "usecond", "3"),
        (1, "void b_kernel(x)", "gpu__time_duration.sum", "nsecond", "1000"),
        (2, "void a_kernel(x)", "gpu__time_duration.sum", "usecond", "4"),
        (3, "void b_kernel(x)", "dram__bytes_read.sum", "byte", "7"),
    ])
    bench.ncu_launches(str(csv))
    lines = capsys.readouterr().out.splitlines()[1:]
    got = {ln.split()[0]: (int(ln.split()[1]), float(ln.split()[2]), float(ln.split()[4])) for ln in lines}
    assert got["a_kernel"] == (2, 7.0, 0.875)
    assert got["b_kernel"] == (1, 1.0, 0.125)
    assert math.isclose(sum(v[2] for v in got.values()), 1.0)

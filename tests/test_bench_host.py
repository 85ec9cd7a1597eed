"""Host-side logic of bench.py: whole-job aggregation (max over ranks, over gloo with two
ranks on the CPU), the reference (CPU oracle) arm's JSON line, peaks and profile lookup."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_aggregate_uses_slowest_rank_and_all_tokens():
    a = bench.aggregate([10.0, 12.5], tokens_per_step_per_rank=425, steps=50, world=2)
    assert a["ms"] == 12.5
    assert a["ms_per_step"] == 12.5 / 50
    assert a["value"] == pytest.approx(2 * 425 * 50 / 0.0125)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    local_ms = 10.0 + 5.0 * rank                    # rank 1 is slower
    t = torch.tensor([local_ms])
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    agg = bench.aggregate([float(t.item())], 100, 4, world)
    q.put((rank, agg))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_with_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    res = dict(q.get(timeout=120) for _ in ps)
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0] == res[1]
    assert res[0]["ms"] == 15.0
    assert res[0]["value"] == pytest.approx(2 * 100 * 4 / 0.015)


def test_reference_arm_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "3"], capture_output=True, text=True, timeout=600,
                         cwd=ROOT)
    assert out.returncode == 0, out.stderr
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC and line["unit"] == "tokens/s"
    assert line["value"] > 0 and line["higher_is_better"] is True
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]


def test_reference_arm_other_ranks_do_nothing(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3"]) == 0
    assert capsys.readouterr().out == ""


def test_peaks_and_profile_lookup(tmp_path, monkeypatch):
    p = bench.load_peaks()
    assert p["source"] in ("measured", "fallback") and p["hbm_gbs"] > 0
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.load_peaks()["source"] == "fallback"
    assert bench.profile_traffic("nothing") is None
    (tmp_path / "profiles").mkdir()
    src = tmp_path / "k.cu"
    src.write_text("kernel")
    import hashlib
    h = hashlib.sha256(b"kernel").hexdigest()
    (tmp_path / "profiles" / "tag.md").write_text(f"traffic_bytes_per_launch: 1234\nsource_sha256: {h} k.cu\n")
    assert bench.profile_traffic("tag") == 1234.0
    src.write_text("changed kernel")
    assert bench.profile_traffic("tag") is None


def test_kernels_per_forward_follows_the_launch_sequence():
    # router; select/permute in one kernel (T*k <= 4096) or four; the row copy for T > 32;
    # then gate_up, down, combine.
    assert [bench.kernels_per_forward(T, 8) for T in (1, 32, 33, 256, 512, 8192)] == \
        [5, 5, 6, 6, 6, 9]
    # the decode path is one kernel
    assert bench.kernels_per_forward(1, 8, "decode") == 1

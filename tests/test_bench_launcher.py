"""bench.py --gpus N starts N ranks itself (one process per GPU) when no
launcher variables are set.  Here the ranks run a CPU stand-in of the per-rank
step (gloo), so the launcher path is checked without a GPU."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_torchrun_argv_shape():
    argv = bench.torchrun_argv(["--gpus", "4", "--steps", "2"], 4, port=29555)
    assert argv[:3] == [sys.executable, "-m", "torch.distributed.run"]
    assert "--nproc-per-node=4" in argv and "--nnodes=1" in argv
    assert argv[argv.index("--master-addr") + 1] == "127.0.0.1"
    assert argv[argv.index("--master-port") + 1] == "29555"
    assert argv[-5] == os.path.join(ROOT, "bench.py")
    assert argv[-4:] == ["--gpus", "4", "--steps", "2"]


@pytest.mark.parametrize("n", [2, 3])
def test_launch_starts_n_gloo_ranks(tmp_path, n):
    probe = os.path.join(ROOT, "tests", "rank_env_probe.py")
    rc = bench.launch([str(tmp_path), "--gpus", str(n)], n, script=probe, timeout_s=120)
    assert rc == 0
    recs = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(n)]
    assert sorted(r["rank"] for r in recs) == list(range(n))
    for r in recs:
        assert r["world"] == n and r["local_rank"] == r["rank"]
        assert r["master_addr"] == "127.0.0.1"
        assert r["sum"] == n * (n + 1) / 2
        assert r["argv"] == ["--gpus", str(n)]


def test_rank_count_mismatch_is_an_error(monkeypatch):
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--gpus", "4"])
    with pytest.raises(SystemExit) as e:
        bench.main()
    assert "4" in str(e.value) and "2 ranks" in str(e.value)

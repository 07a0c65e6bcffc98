"""Host-side checks of the in-tree build: processes that build at once (one
per GPU under a multi-rank launch) must not compile over one another."""
import multiprocessing as mp
import os
import time


def _child(marker: str, log: str) -> None:
    from mixture_experts_ffn_09_b200 import build as b

    b.up_to_date = lambda: os.path.exists(marker)

    def fake(verbose: bool) -> str:
        with open(log, "a") as f:
            f.write(f"start {os.getpid()} {time.time()}\n")
        time.sleep(0.3)
        open(marker, "w").close()
        with open(log, "a") as f:
            f.write(f"end {os.getpid()} {time.time()}\n")
        return b.LIB

    b._build_locked = fake
    assert b.build() == b.LIB


def test_concurrent_builds_compile_once(tmp_path):
    marker, log = str(tmp_path / "built"), str(tmp_path / "log")
    ctx = mp.get_context("spawn")
    ps = [ctx.Process(target=_child, args=(marker, log)) for _ in range(3)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(120)
        assert p.exitcode == 0
    lines = open(log).read().split()
    assert lines.count("start") == 1 and lines.count("end") == 1


def test_library_is_current_after_build():
    from mixture_experts_ffn_09_b200 import build as b

    b.build()
    assert b.up_to_date()

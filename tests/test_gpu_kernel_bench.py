"""The single-entry-point driver (two_sided_adaptive_bakron_b200.kernel_bench) runs every
operation on a small workload (B200): the commands under profiles/ use it."""
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("args", [["--op", "ldl", "--d", "300"], ["--op", "round"],
                                  ["--op", "loss"], ["--op", "gram", "--k", "512"],
                                  ["--op", "sketch_b", "--k", "4"], ["--op", "rht"]])
def test_kernel_bench_runs(args, capsys):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from two_sided_adaptive_bakron_b200 import build, kernel_bench
    build.build()
    assert kernel_bench.main(args + ["--workload", "small_64x128", "--iters", "2"]) == 0
    assert " ms (mean of 1)" in capsys.readouterr().out

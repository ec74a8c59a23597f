"""The Python example of README.md runs as written (its code block is executed)."""
import os
import re

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_readme_python_example_runs():
    with open(os.path.join(ROOT, "README.md")) as f:
        text = f.read()
    code = re.search(r"```python\n(.*?)```", text, re.S).group(1)
    env = {}
    exec(compile(code, "README.md", "exec"), env)
    hq, torch = env["hq"], env["torch"]
    torch.cuda.synchronize()
    assert hq.read_stats(env["codec"].stats)["status"] == 0
    assert abs(env["cal"]["bps"] - 4.0) <= 0.002
    assert env["s"].shape == (32, 256) and bool(torch.isfinite(env["s"]).all())
    assert hq.read_stats(env["rcache"].stats)["status"] == 0 and env["rcache"].tokens == 256
    # the batch decodes to what single calls give
    Ws, Ws_hat, p = env["Ws"], env["Ws_hat"], env["p"]
    one = hq.Codec(1024, 4096, p)
    ref = one.dequantize(one.quantize(Ws[5]), torch.empty_like(Ws[5]))
    torch.cuda.synchronize()
    assert torch.equal(Ws_hat[5], ref)

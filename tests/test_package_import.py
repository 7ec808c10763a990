"""The package without its CUDA library (a clean checkout): the build step and
the input generators import, and the binding refuses to load -- there is no
fallback path."""
import os
import shutil
import subprocess
import sys

import chunked_block_self_b200

PKG = os.path.dirname(os.path.abspath(chunked_block_self_b200.__file__))


def _run(code, root):
    env = dict(os.environ, PYTHONPATH=root)
    return subprocess.run([sys.executable, "-c", code], cwd=root, env=env, capture_output=True, text=True,
                          timeout=300)


def test_clean_checkout_imports(tmp_path):
    dst = tmp_path / "chunked_block_self_b200"
    dst.mkdir()
    for f in os.listdir(PKG):
        if f.endswith(".py"):
            shutil.copy(os.path.join(PKG, f), dst / f)
    assert not (dst / "libnle.so").exists()
    ok = _run("from chunked_block_self_b200 import build, workloads\n"
              "import chunked_block_self_b200 as p\n"
              "assert callable(build.build) and callable(workloads.cu_seqlens)\n"
              "assert p.workloads is workloads\n", str(tmp_path))
    assert ok.returncode == 0, ok.stderr
    bad = _run("import chunked_block_self_b200.nle", str(tmp_path))
    assert bad.returncode != 0 and "libnle.so not found" in bad.stderr

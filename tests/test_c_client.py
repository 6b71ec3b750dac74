"""The boundary from plain C: tests/c_abi_client.c includes include/hisa.h,
compiles as strict C11 (-pedantic, warnings as errors), links the built
library and checks workspace sizes and argument rejections, none of which
needs a GPU."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "hierarchical_top_indexer_b200")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_client_compiles_links_and_passes(tmp_path):
    from tests.test_abi import build_module
    build = build_module()
    if build.stale():
        build.build()
    exe = str(tmp_path / "c_abi_client")
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c_abi_client.c"),
                    "-L", PKG, "-lhisa_b200", f"-Wl,-rpath,{PKG}", "-o", exe], check=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == "c abi ok"

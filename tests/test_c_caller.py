"""The boundary is a C ABI: a plain C99 program includes include/smla.h
(compiled with -std=c99 -pedantic -Werror), links libsmla.so and calls the
entry points that need no GPU: the version, the status strings, the NSPLIT
heuristic, the workspace sizes, and argument checks that fail before any
launch.  Its answers must equal the ones the Python binding gets."""
import os
import shutil
import subprocess

import pytest

from sparse_mla_decode_partial_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "sparse_mla_decode_partial_b200")

C_PROGRAM = r"""
#include <stdio.h>
#include "smla.h"

int main(void) {
    int fake[64] = {0};
    const void *p = fake;
    /* a bad page size is refused before anything is launched */
    smla_status bad_page = smla_decode(p, p, 1, (const int32_t *)p, 1, (const int32_t *)p,
                                       1, 1, 16, 4, 16, 0.1f, 1, NULL, 0, (void *)fake,
                                       (float *)fake, NULL);
    /* an empty problem is legal and launches nothing */
    smla_status empty = smla_decode(NULL, NULL, 0, NULL, 0, NULL, 0, 1, 16, 4, SMLA_PAGE_SIZE,
                                    0.1f, 1, NULL, 0, NULL, NULL, NULL);
    printf("version %d\n", smla_version());
    printf("nsplit %d %d %d\n", smla_choose_nsplit(1, 1, 16, 2048, 148),
           smla_choose_nsplit(64, 1, 16, 2048, 148), smla_choose_nsplit(60, 1, 64, 2048, 148));
    printf("workspace %zu %zu\n", smla_workspace_bytes(2, 3, 16, 4),
           smla_workspace_host_bytes(1, 1, 16, 2048, 1024, 64));
    printf("dense %d %zu\n", smla_dense_nsplit(1, 9, 8, 46089),
           smla_dense_workspace_bytes(1, 9, 8, 46089, 74));
    printf("indexer %zu %zu\n", smla_indexer_workspace_bytes(60, 1, 131072),
           smla_indexer_select_workspace_bytes(60, 1, 131072));
    printf("status %d %d\n", (int)bad_page, (int)empty);
    printf("string %s\n", smla_status_string(SMLA_ERR_MISALIGNED));
    return 0;
}
"""


@pytest.fixture(scope="module")
def c_caller(tmp_path_factory):
    if shutil.which("gcc") is None:
        pytest.skip("gcc is not installed")
    build.build()
    d = tmp_path_factory.mktemp("c_caller")
    src, exe = d / "caller.c", d / "caller"
    src.write_text(C_PROGRAM)
    subprocess.run(["gcc", "-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror",
                    "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                    "-L", PKG, "-lsmla", f"-Wl,-rpath,{PKG}"], check=True,
                   capture_output=True, text=True)
    env = dict(os.environ)
    env.pop("SMLA_NSPLIT", None)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120, env=env)
    assert r.returncode == 0, r.stderr
    return dict(line.split(" ", 1) for line in r.stdout.splitlines())


def test_c_program_sees_what_the_binding_sees(c_caller, monkeypatch):
    monkeypatch.delenv("SMLA_NSPLIT", raising=False)
    lib = binding.lib()
    assert int(c_caller["version"]) == lib.smla_version()
    assert [int(x) for x in c_caller["nsplit"].split()] == [
        binding.choose_nsplit(1, 1, 16, 2048, 148), binding.choose_nsplit(64, 1, 16, 2048, 148),
        binding.choose_nsplit(60, 1, 64, 2048, 148)]
    assert [int(x) for x in c_caller["workspace"].split()] == [
        binding.workspace_bytes(2, 3, 16, 4), binding.workspace_host_bytes(1, 1, 16, 2048, 1024, 64)]
    assert [int(x) for x in c_caller["dense"].split()] == [
        binding.dense_nsplit(1, 9, 8, 46089), binding.dense_workspace_bytes(1, 9, 8, 46089, 74)]
    assert [int(x) for x in c_caller["indexer"].split()] == [
        binding.indexer_workspace_bytes(60, 1, 131072),
        binding.indexer_select_workspace_bytes(60, 1, 131072)]


def test_c_program_gets_status_codes_before_any_launch(c_caller):
    bad_page, empty = (int(x) for x in c_caller["status"].split())
    assert binding.STATUS[bad_page] == "SMLA_ERR_UNSUPPORTED"
    assert binding.STATUS[empty] == "SMLA_OK"
    assert c_caller["string"].startswith("SMLA_ERR_MISALIGNED")

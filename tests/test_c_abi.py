"""The boundary from plain C (CPU): a C99 program that includes include/pwp.h and links
libpwp.so compiles without warnings, and its host-only calls (version, status strings,
workspace sizing, argument checks) behave as the header states -- no GPU needed."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIBDIR = os.path.join(ROOT, "post_weight_pruning_b200")

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "pwp.h"

int main(void) {
    pwp_config cfg = {PWP_THANOS, PWP_UNSTRUCTURED, 0, 0, 0.5f, 128, 0.01f, 0.0f};
    size_t ws = pwp_workspace_bytes(&cfg, 4096, 4096);
    pwp_config nm = {PWP_THANOS, PWP_NM, 2, 4, 0.0f, 128, 0.01f, 0.0f};
    pwp_config bad = {PWP_THANOS, PWP_NM, 3, 6, 0.0f, 128, 0.01f, 0.0f};       /* m not a power of two */
    pwp_config wanda = {PWP_WANDA, PWP_UNSTRUCTURED, 0, 0, 0.5f, 0, 0.0f, 0.0f}; /* block ignored */
    char W[16];
    printf("version %d\n", (int)pwp_version());
    printf("ws %zu\n", ws);
    printf("ws_nm %zu\n", pwp_workspace_bytes(&nm, 4096, 4096));
    printf("ws_bad %zu\n", pwp_workspace_bytes(&bad, 4096, 4096));
    printf("ws_wanda %zu\n", pwp_workspace_bytes(&wanda, 4096, 4096));
    printf("einval %d\n", (int)pwp_prune_layer(&cfg, NULL, PWP_BF16, 16, 16, NULL, NULL, NULL, NULL, 0,
                                                NULL, NULL));
    printf("eworkspace %d\n", (int)pwp_prune_layer(&cfg, W, PWP_BF16, 16, 16, (float*)W, (float*)W,
                                                    (uint8_t*)W, NULL, 0, (pwp_stats*)W, NULL));
    printf("status %s\n", pwp_status_string(PWP_ENOTSPD));
    printf("stats %zu\n", sizeof(pwp_stats));
    printf("config %zu\n", sizeof(pwp_config));
    return 0;
}
"""


@pytest.fixture(scope="module")
def program(tmp_path_factory):
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    if not os.path.exists(os.path.join(LIBDIR, "libpwp.so")):
        pytest.skip("libpwp.so not built")
    d = tmp_path_factory.mktemp("c_abi")
    src, exe = d / "main.c", d / "main"
    src.write_text(PROGRAM)
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I",
                        os.path.join(ROOT, "include"), str(src), "-o", str(exe), "-L", LIBDIR, "-lpwp",
                        "-Wl,-rpath," + LIBDIR], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stderr
    return dict(line.split(" ", 1) for line in out.stdout.strip().splitlines())


def test_header_is_plain_c_and_host_calls_work(program):
    import ctypes
    import post_weight_pruning_b200 as pwp
    assert int(program["version"]) == pwp.lib().pwp_version()
    assert int(program["ws"]) > 0 and int(program["ws_nm"]) > 0 and int(program["ws_wanda"]) > 0
    assert int(program["ws_bad"]) == 0
    assert int(program["ws"]) == pwp.workspace_bytes(pwp.config(), 4096, 4096)
    assert int(program["einval"]) == 1
    assert int(program["eworkspace"]) == 3
    assert program["status"] == "damped Hessian is not positive definite"
    assert int(program["stats"]) == ctypes.sizeof(pwp.Stats)
    assert int(program["config"]) == ctypes.sizeof(pwp.Config)

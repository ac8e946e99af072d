"""The boundary from plain C: a C11 program that includes only
include/spec_verify.h and links libspecverify.so (no torch, no Python)
queries workspace sizes and status strings and gets the documented host-side
errors back.  Nothing here touches a GPU: every call fails validation before
any CUDA call, or returns early for an empty batch."""
import os
import subprocess

from speculative_decoding_verification_88_b200 import build as svbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CLIENT = r"""
#include <stdio.h>
#include <string.h>
#include "spec_verify.h"

static unsigned char buf[4096] __attribute__((aligned(16)));

int main(void) {
    int bad = 0;
    size_t ws = spec_verify_workspace_size(256, 1, 8, 128256);
    if (ws == 0 || ws % 256 != 0) { printf("workspace size %zu\n", ws); bad = 1; }
    if (spec_verify_workspace_size(1, 1, 33, 10) != 0) { printf("k limit\n"); bad = 1; }
    if (spec_verify_tree_stochastic_workspace_size(64, 26, 128256) == 0) { printf("tree ws\n"); bad = 1; }
    if (strncmp(spec_verify_status_string(SV_ERR_WORKSPACE), "SV_ERR_WORKSPACE", 16) != 0) {
        printf("status %s\n", spec_verify_status_string(SV_ERR_WORKSPACE)); bad = 1;
    }
    /* temperature 0: rejected on the host */
    int r = spec_verify_stochastic(buf, SV_BF16, 40, 8, buf, SV_BF16, 32, 8, (const int32_t *)buf,
                                   4, 4, 8, 0.0f, 1, 0, (int32_t *)buf, (int32_t *)buf, NULL,
                                   buf, sizeof buf, NULL);
    if (r != SV_ERR_INVALID_ARG) { printf("temperature -> %d\n", r); bad = 1; }
    /* misaligned accepted_len */
    r = spec_verify_greedy(buf, SV_BF16, 40, 8, (const int32_t *)buf, 4, 4, 8,
                           (int32_t *)(buf + 1), (int32_t *)buf, buf, sizeof buf, NULL);
    if (r != SV_ERR_MISALIGNED) { printf("misaligned -> %d\n", r); bad = 1; }
    /* workspace too small */
    r = spec_verify_tree_stochastic(buf, SV_BF16, 80, 8, (const int32_t *)buf,
                                    (const int32_t *)buf, 2, 10, 8, 1.0f, 3, 0, (int32_t *)buf,
                                    (int32_t *)buf, (int32_t *)buf, buf, 64, NULL);
    if (r != SV_ERR_WORKSPACE) { printf("workspace -> %d\n", r); bad = 1; }
    /* empty batch: nothing to do */
    r = spec_verify_tree_greedy(NULL, SV_BF16, 0, 0, NULL, NULL, 0, 4, 8, NULL, NULL, NULL,
                                NULL, 0, NULL);
    if (r != SV_OK) { printf("empty -> %d\n", r); bad = 1; }
    puts(bad ? "FAIL" : "OK");
    return bad;
}
"""


def test_plain_c_client_links_and_calls_the_library(tmp_path):
    lib = svbuild.build()
    src = tmp_path / "client.c"
    src.write_text(CLIENT)
    exe = tmp_path / "client"
    libdir = os.path.dirname(lib)
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Werror", f"-I{os.path.join(ROOT, 'include')}",
                    str(src), "-o", str(exe), f"-L{libdir}", "-lspecverify",
                    f"-Wl,-rpath,{libdir}"], check=True)
    p = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert p.returncode == 0 and p.stdout.strip().endswith("OK"), p.stdout + p.stderr

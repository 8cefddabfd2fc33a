"""The boundary from plain C: a C99 program that includes include/tq.h, links
libtq.so and calls the host-only entry points (no GPU needed).  It checks
the ABI version, a codebook against its stated properties (ascending
centroids, midpoint boundaries, symmetry), the cache byte sizes of a K4/V2
layer with a 64-bit sketch, and that a paged call rejects a block size that
is not a multiple of 16 before touching the device."""

import os
import shutil
import subprocess

import pytest

from conftest import ROOT

C_SOURCE = r"""
#include <math.h>
#include <stdio.h>
#include "tq.h"

int main(void) {
    if (tq_abi_version() != TQ_ABI_VERSION) return 1;
    tq_codebook cb;
    if (tq_codebook_init(128, 3, &cb) != TQ_OK) return 2;
    for (int j = 0; j + 1 < 8; ++j) {
        if (!(cb.centroids[j] < cb.centroids[j + 1])) return 3;
        if (fabs(cb.boundaries[j] - 0.5 * (cb.centroids[j] + cb.centroids[j + 1])) > 1e-15) return 4;
        if (cb.centroids[j] != -cb.centroids[7 - j]) return 5;
    }
    tq_params p = {0};
    p.head_dim = 128; p.num_q_heads = 32; p.num_kv_heads = 8;
    p.k_mode = TQ_MODE_TURBO; p.v_mode = TQ_MODE_TURBO; p.k_bits = 4; p.v_bits = 2;
    p.qjl_dims = 64; p.seed = 7;
    size_t sizes[6];
    if (tq_cache_bytes(&p, 2, 1024, sizes) != TQ_OK) return 6;
    const size_t slots = 2u * 8u * 1024u;
    if (sizes[0] != slots * 64 || sizes[1] != slots * 2 || sizes[2] != slots * 8 || sizes[3] != slots * 2 ||
        sizes[4] != slots * 32 || sizes[5] != slots * 2)
        return 7;
    tq_codebook kcb, vcb;
    p.qjl_dims = 0;
    if (tq_codebook_init(128, 4, &kcb) != TQ_OK || tq_codebook_init(128, 2, &vcb) != TQ_OK) return 8;
    static char fake[64] __attribute__((aligned(16)));
    tq_cache pool = {8, 24, (uint8_t*)fake, (uint16_t*)fake, 0, 0, (uint8_t*)fake, (uint16_t*)fake, 0};
    tq_block_table table = {(const int32_t*)fake, 2, 4};
    if (tq_quantize_append_paged(&p, &kcb, &vcb, fake, fake, TQ_BF16, 1, (const int32_t*)fake, &pool, &table,
                                 0, 0) != TQ_ERR_INVALID_ARG)
        return 9;
    printf("%s\n", tq_status_string(TQ_ERR_INVALID_ARG));
    return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_plain_c_program_uses_the_library(tmp_path):
    pkg = os.path.join(ROOT, "bit_kv_cache_tq_b200")
    src = tmp_path / "use_tq.c"
    exe = tmp_path / "use_tq"
    src.write_text(C_SOURCE)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe), "-L", pkg, "-l:libtq.so", "-Wl,-rpath," + pkg, "-lm"],
                   check=True, capture_output=True, text=True)
    res = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert res.returncode == 0, (res.returncode, res.stdout, res.stderr)
    assert res.stdout.strip(), res.stdout

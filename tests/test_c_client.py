"""A plain C program compiled against include/gdn.h and linked with libgdn.so calls the
boundary directly (no Python in between). Only host-side validation paths run, so no GPU is
needed: every call below must be rejected before any CUDA work."""
import os
import shutil
import subprocess
import textwrap

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

C_SRC = textwrap.dedent(r"""
    #include <stdio.h>
    #include <string.h>
    #include "gdn.h"

    static int fails = 0;
    static void expect(const char *what, gdn_status_t got, gdn_status_t want) {
        if (got != want) { printf("FAIL %s: %s (want %s)\n", what, gdn_status_str(got), gdn_status_str(want)); ++fails; }
    }

    int main(void) {
        void *p = (void *)0x10000;   /* aligned, never dereferenced: validation fails first */
        float *f = (float *)p;
        gdn_fwd_opts_t opts;
        memset(&opts, 0, sizeof(opts));
        if (gdn_version() < 100) { printf("FAIL version\n"); ++fails; }
        if (strcmp(gdn_status_str(GDN_ERR_TIMEOUT), "GDN_ERR_TIMEOUT") != 0) { printf("FAIL names\n"); ++fails; }
        expect("la B=0", lin_attn_chunk_fwd(p, p, p, NULL, f, NULL, NULL, 0, 1, 8, 64, 64, 64, 1.f, GDN_BF16, NULL),
               GDN_ERR_INVALID_ARG);
        expect("gdn without beta", gdn_chunk_fwd(p, p, p, NULL, NULL, f, NULL, NULL, 1, 1, 8, 64, 64, 64, 1.f, GDN_BF16, NULL),
               GDN_ERR_INVALID_ARG);
        expect("gdn dk=96", gdn_chunk_fwd(p, p, p, f, NULL, f, NULL, NULL, 1, 1, 8, 96, 64, 64, 1.f, GDN_BF16, NULL),
               GDN_ERR_UNSUPPORTED);
        expect("varlen no offsets", gdn_chunk_fwd_varlen(p, p, p, f, NULL, f, NULL, NULL, NULL, 2, 1, 8, 64, 64, 64, 1.f,
                                                         GDN_BF16, NULL), GDN_ERR_INVALID_ARG);
        opts.out_dtype = (gdn_dtype_t)7;
        expect("ex bad out_dtype", gdn_chunk_fwd_ex(p, p, p, f, NULL, p, NULL, NULL, NULL, 1, 1, 8, 64, 64, 64, 1.f, GDN_BF16,
                                                    &opts, NULL), GDN_ERR_INVALID_ARG);
        opts.out_dtype = GDN_BF16;
        opts.g_per_key = 2;
        expect("ex bad g_per_key", lin_attn_chunk_fwd_ex(p, p, p, NULL, p, NULL, NULL, NULL, 1, 1, 8, 64, 64, 64, 1.f,
                                                         GDN_BF16, &opts, NULL), GDN_ERR_INVALID_ARG);
        opts.g_per_key = 0;
        opts.d_skip = (const float *)((char *)p + 2);
        expect("ex misaligned d_skip", gdn_chunk_fwd_ex(p, p, p, f, NULL, p, NULL, NULL, NULL, 1, 1, 8, 64, 64, 64, 1.f,
                                                        GDN_BF16, &opts, NULL), GDN_ERR_INVALID_ARG);
        expect("decode N=0", gdn_decode_step(p, p, p, NULL, NULL, f, f, 0, 1, 64, 64, 1.f, GDN_BF16, NULL),
               GDN_ERR_INVALID_ARG);
        expect("decode_ex dk=32", gdn_decode_step_ex(p, p, p, NULL, NULL, f, p, 1, 1, 32, 64, 1.f, GDN_BF16, NULL, NULL),
               GDN_ERR_UNSUPPORTED);
        printf(fails ? "c client: %d failures\n" : "c client ok\n", fails);
        return fails != 0;
    }
""")


def test_c_program_links_and_validates(tmp_path):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    from gated_deltanet_sequence_b200 import build
    lib = build.build()
    libdir = os.path.dirname(lib)
    src = tmp_path / "client.c"
    src.write_text(C_SRC)
    exe = tmp_path / "client"
    cuda_lib = "/usr/local/cuda/lib64"
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
                           "-o", str(exe), "-L", libdir, "-lgdn", f"-Wl,-rpath,{libdir}", f"-Wl,-rpath,{cuda_lib}"])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "c client ok" in out.stdout

"""The boundary is plain C: a C99 program (and the same file as C++) that
includes include/qstate.h compiles with every warning an error, links
libqstate.so and gets the documented answers from calls that need no GPU
(NULL objects, invalid and unsupported layouts, error strings, the kernel
name of no object)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "bit_recurrent_state_decode_b200")

CLIENT = r"""
#include <stdio.h>
#include <string.h>
#include "qstate.h"

int main(void) {
    qstate_layout L;
    qstate* s = NULL;
    qstate_sizes z;
    int rc;
    if (qstate_create(NULL, 4, 64, QSTATE_DYNAMIC, QSTATE_RTN, 0.0f, &s) != QSTATE_EINVAL) return 1;
    if (qstate_step(NULL, NULL, NULL, NULL, NULL, NULL, NULL) != QSTATE_EINVAL) return 2;
    if (qstate_dequant(NULL, NULL, NULL) != QSTATE_EINVAL) return 3;
    if (qstate_get_sizes(NULL, &z) != QSTATE_EINVAL) return 4;
    if (qstate_set_lrb(NULL, 1, 15, 0.5f) != QSTATE_EINVAL) return 5;
    if (qstate_kernel(NULL)[0] != '\0') return 6;
    if (strlen(qstate_error_string(QSTATE_ENOMEM)) == 0) return 7;
    memset(&L, 0, sizeof L);
    L.batch = 1;
    L.heads = 2;
    L.d_k = 96;                     /* not built: d_k in {64, 128} */
    L.d_v = 64;
    L.layers = 1;
    L.kind = QSTATE_RETNET;
    L.gamma = 0.96875f;
    L.qkv_dtype = QSTATE_F32;
    L.gate_dtype = QSTATE_F32;
    L.scale_dtype = QSTATE_F16;
    rc = qstate_create(&L, 4, 64, QSTATE_DYNAMIC, QSTATE_RTN, 0.0f, &s);
    if (rc != QSTATE_EUNSUPPORTED || s != NULL) return 8;
    L.d_k = 64;
    rc = qstate_create(&L, 5, 64, QSTATE_DYNAMIC, QSTATE_RTN, 0.0f, &s);   /* 5-bit codes */
    if (rc != QSTATE_EINVAL || s != NULL) return 9;
    puts("c client ok");
    return 0;
}
"""


@pytest.mark.parametrize("lang", ["c", "c++"])
def test_c_client_builds_links_and_runs(tmp_path, lang):
    from bit_recurrent_state_decode_b200 import build
    build.build()
    cc = shutil.which("gcc" if lang == "c" else "g++")
    if cc is None:
        pytest.skip("no host compiler")
    src = tmp_path / ("client.c" if lang == "c" else "client.cpp")
    src.write_text(CLIENT)
    exe = tmp_path / "client"
    std = ["-std=c99"] if lang == "c" else ["-std=c++17"]
    subprocess.run([cc, *std, "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    "-o", str(exe), str(src), "-L", PKG, "-lqstate", f"-Wl,-rpath,{PKG}"],
                   check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and "c client ok" in r.stdout, (r.returncode, r.stdout, r.stderr)


def test_readme_c_example_compiles(tmp_path):
    """The C example in README.md, placed in a function whose parameters are
    the buffers it names, compiles against the header as C99 with every
    warning an error (its field names and calls are the header's)."""
    cc = shutil.which("gcc")
    if cc is None:
        pytest.skip("no host compiler")
    text = open(os.path.join(ROOT, "README.md")).read()
    start = text.index("```c\n") + len("```c\n")
    body = text[start:text.index("```", start)]
    lines = [l for l in body.splitlines() if not l.startswith("#include")]
    src = tmp_path / "readme_example.c"
    src.write_text(
        "#include <stdio.h>\n#include \"qstate.h\"\n"
        "void example(const void* q, const void* k, const void* v, const void* gates, float* out,\n"
        "             float* S_hat, qstate_stream stream) {\n"
        + "\n".join("    " + l for l in lines) + "\n    (void)rc;\n}\n"
        "int main(void) { return 0; }\n")
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I",
                        os.path.join(ROOT, "include"), "-c", str(src), "-o",
                        str(tmp_path / "readme_example.o")], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr

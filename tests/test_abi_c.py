"""The boundary is a C ABI: include/mom.h compiles as strict C99, a C program
links against libmom_b200.so and resolves every declared entry point, and the
host-side checks answer from C exactly as from Python.  Nothing here touches
a GPU (the calls fail validation before any launch), so it runs on the CPU.
"""
import os
import re
import shutil
import subprocess

import pytest

from tests.conftest import ROOT

HEADER_DIR = os.path.join(ROOT, "include")
PKG = os.path.join(ROOT, "mixture_memories_layer_b200")


def _declared():
    text = open(os.path.join(HEADER_DIR, "mom.h")).read()
    return sorted(set(re.findall(r"^(?:mom_status|size_t|uint64_t|const char\*)\s+(mom_\w+)\s*\(", text, re.M)))


C_MAIN = r"""
#include <stdio.h>
#include <string.h>
#include "mom.h"

typedef void (*any_fn)(void);
static const any_fn every_entry[] = { %(entries)s };

int main(void) {
    void* fake = (void*)0x10000;     /* never dereferenced: validation fails first */
    int bad = 0;
    for (size_t i = 0; i < sizeof(every_entry) / sizeof(every_entry[0]); ++i)
        if (!every_entry[i]) bad |= 1;
    if (strcmp(mom_status_string(MOM_ERR_UNSUPPORTED), "unsupported shape or type") != 0) bad |= 2;
    if (mom_permute_workspace_size(1000, 2, 4, 3) < MOM_WS_HEADER_BYTES) bad |= 4;
    /* top_k > n_mem */
    if (mom_router_topk(fake, fake, NULL, MOM_BF16, 10, 64, 4, 5, fake, fake, NULL, NULL) != MOM_ERR_ARG) bad |= 8;
    /* n_tok * top_k = 2^31 */
    if (mom_permute(fake, (int64_t)1 << 30, 2, 4, fake, 1, fake, fake, fake, fake, fake, 1 << 20, NULL)
        != MOM_ERR_UNSUPPORTED) bad |= 16;
    /* head dimension 96 */
    if (mom_kv_proj_grouped(fake, fake, fake, fake, fake, fake, fake, fake, MOM_BF16, 10, 256, 2, 96, 4, 2,
                            fake, fake, fake, fake, fake, fake, fake, fake, 4096, NULL) != MOM_ERR_UNSUPPORTED)
        bad |= 32;
    printf("entries %%d bad %%d\n", (int)(sizeof(every_entry) / sizeof(every_entry[0])), bad);
    return bad;
}
"""


@pytest.fixture(scope="module")
def lib_path():
    from mixture_memories_layer_b200 import build
    return build.build(verbose=False)


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_program_links_and_validates(lib_path):
    names = _declared()
    work = os.path.join(PKG, "_build", "c_abi_check")      # build scratch, git-ignored
    os.makedirs(work, exist_ok=True)
    src = os.path.join(work, "use_mom.c")
    with open(src, "w") as fh:
        fh.write(C_MAIN % {"entries": ", ".join("(any_fn)%s" % n for n in names)})
    exe = os.path.join(work, "use_mom")
    libdir = os.path.dirname(lib_path)
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
           "-I", HEADER_DIR, str(src), "-o", str(exe), "-L", libdir, "-lmom_b200", "-Wl,-rpath," + libdir]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, (run.stdout, run.stderr)
    assert run.stdout.strip() == "entries %d bad 0" % len(names)

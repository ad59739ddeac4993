"""The C-ABI library loads and exports every function include/*.h declares
(no GPU needed; no compute calls)."""
import glob
import os
import re
import subprocess

import pytest

from tests.conftest import ROOT


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^[A-Za-z_][\w \*]*?\b(pa_\w+)\s*\(", text, flags=re.M):
            names.add(m.group(1))
    return sorted(names)


@pytest.fixture(scope="module")
def built_lib():
    from paged_kv_cache_326_b200 import build
    return build.build()


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("pa_kv_cache_write", "pa_paged_attn_decode",
                     "pa_paged_attn_decode_workspace_size", "pa_status_string",
                     "pa_bm_create", "pa_bm_destroy", "pa_bm_add_seq", "pa_bm_fork",
                     "pa_bm_append_slot", "pa_bm_free_seq", "pa_bm_num_free",
                     "pa_bm_refcount", "pa_bm_export"):
        assert required in names


def test_library_exports_every_declared_symbol(built_lib):
    out = subprocess.run(["nm", "-D", "--defined-only", built_lib], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing


def test_library_loads_and_binds(built_lib):
    import paged_kv_cache_326_b200 as P
    lib = P.lib()
    for n in declared_functions():
        assert hasattr(lib, n)
    assert P.pa_status_string(0) == "ok"
    assert P.pa_status_string(-10) == "bounded wait gave up"


def test_binding_refuses_cpu_tensors(built_lib):
    import torch
    import paged_kv_cache_326_b200 as P
    q = torch.zeros(1, 1, 64, dtype=torch.float16)
    kc = torch.zeros(1, 1, 4, 64, dtype=torch.float16)
    with pytest.raises(TypeError):
        P.pa_kv_cache_write(q, q, kc, kc, torch.zeros(1, dtype=torch.int64))


def test_invalid_arguments_are_rejected_before_launch(built_lib):
    """Null pointers and unsupported sizes return PA_ERR_INVALID without
    touching a GPU."""
    import paged_kv_cache_326_b200 as P
    lib = P.lib()
    assert lib.pa_kv_cache_write(None, None, None, None, None, 1, 8, 64, 4, 64, 0, None,
                                 None) == P.binding.PA_ERR_INVALID
    assert lib.pa_kv_cache_write(None, None, None, None, None, 1, 8, 96, 4, 64, 0, None,
                                 None) == P.binding.PA_ERR_INVALID
    assert lib.pa_paged_attn_decode(None, None, None, None, None, None, 1.0, 4, 8, 64, 4, 8, 64,
                                    0, None, 0, None, None) == P.binding.PA_ERR_INVALID
    assert lib.pa_paged_attn_decode(None, None, None, None, None, None, 1.0, 4, 8, 100, 4, 8, 64,
                                    0, None, 0, None, None) == P.binding.PA_ERR_INVALID
    assert lib.pa_set_option(99, 0) == P.binding.PA_ERR_INVALID


def test_header_is_plain_c(tmp_path):
    """include/pagedattn.h compiles as strict C99 with every warning an error."""
    src = tmp_path / "use.c"
    src.write_text('#include "pagedattn.h"\nint main(void) { return PA_OK; }\n')
    res = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                          f"-I{os.path.join(ROOT, 'include')}", "-c", str(src), "-o",
                          str(tmp_path / "use.o")], capture_output=True, text=True)
    assert res.returncode == 0, res.stderr


def test_plain_c_program_uses_the_host_calls(tmp_path, built_lib):
    """A C99 program links libpagedattn.so and drives the block manager,
    prefix reuse and the shared-prefix splitter (no GPU needed)."""
    exe = tmp_path / "c_abi_host"
    lib_dir = os.path.dirname(built_lib)
    res = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                          f"-I{os.path.join(ROOT, 'include')}",
                          os.path.join(ROOT, "tests", "c_abi_host.c"), "-o", str(exe),
                          f"-L{lib_dir}", "-l:libpagedattn.so", f"-Wl,-rpath,{lib_dir}"],
                         capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0 and run.stdout.strip() == "ok", run.stderr

"""The C-ABI library loads and exports every symbol include/dg.h declares (no GPU needed).

Also checks that the ctypes struct matches the C header's layout (compiled with
gcc) and that dg_workspace_bytes validates configurations on the host.
"""
import ctypes
import os
import re
import subprocess

import pytest

import synthetic
import uniform_state_text_b200 as dg
from uniform_state_text_b200 import build as dgbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dg.h")


@pytest.fixture(scope="module")
def lib():
    dgbuild.build()
    return dg.lib()


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s+(dg_[a-z_0-9]+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = _declared_functions()
    assert len(names) >= 12, names
    out = subprocess.run(["nm", "-D", "--defined-only", dg.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r" T (dg_[a-z_0-9]+)$", out, flags=re.M))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        assert hasattr(lib, n)


def test_struct_layout_matches_header(tmp_path):
    prog = tmp_path / "layout.c"
    fields = [f[0] for f in dg.dg_config._fields_]
    body = "\n".join(f'  printf("{f} %zu\\n", offsetof(dg_config, {f}));' for f in fields)
    prog.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "dg.h"\nint main(void){\n'
                    '  printf("size %zu\\n", sizeof(dg_config));\n' + body + "\n  return 0;\n}\n")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c11", "-I", os.path.dirname(HEADER), str(prog), "-o", str(exe)],
                   check=True)
    got = dict(line.split() for line in subprocess.run([str(exe)], capture_output=True, text=True,
                                                       check=True).stdout.splitlines())
    assert int(got["size"]) == ctypes.sizeof(dg.dg_config)
    for f in fields:
        assert int(got[f]) == getattr(dg.dg_config, f).offset, f


def _cfg(**kw):
    return dg.make_config(synthetic.TINY.replace(**kw))


def test_workspace_bytes_valid_configs(lib):
    for w in synthetic.WORKLOADS.values():
        n = dg.dg_workspace_bytes(dg.make_config(w, dg.DG_IMPL_SIMT))
        assert n > w.C * w.d * 4
        assert n % 256 == 0


@pytest.mark.parametrize("kw", [dict(V=1000), dict(V=32), dict(C=0), dict(C=2048), dict(d=12),
                                dict(max_steps=0), dict(T_start=0.0), dict(tau=-1.0),
                                dict(stop_unchanged=0), dict(stop_rule=5), dict(accept_rule=2),
                                dict(tau=float("inf")), dict(T_end=float("nan")),
                                dict(token_rule=2), dict(canvases=3), dict(canvases=-1),
                                dict(canvases=128, C=128)])
def test_workspace_bytes_rejects_invalid(lib, kw):
    assert dg.dg_workspace_bytes(_cfg(**kw)) == 0


def test_canvases_and_draw_options_are_accepted(lib):
    for kw in (dict(canvases=1), dict(canvases=4), dict(canvases=16), dict(token_rule=1)):
        assert dg.dg_workspace_bytes(_cfg(**kw)) > 0


@pytest.mark.parametrize("shard", [(0, 1024), (512, 4096), (300, 512), (0, 0 + 1)])
def test_vocabulary_shard_bounds(lib, shard):
    w = synthetic.SMALL.replace(C=128, V=4096, d=256)
    cfg = dg.make_config(w, dg.DG_IMPL_AUTO, shard=shard)
    v0, nv = shard
    ok = v0 % 256 == 0 and nv % 256 == 0 and nv > 0 and v0 + nv <= w.V
    assert (dg.dg_workspace_bytes(cfg) > 0) == ok
    # a shard needs the tensor-core kernels; the partials buffer exists only then
    assert (dg.dg_partials_bytes(cfg) > 0) == ok
    if ok:
        assert dg.dg_partials_bytes(cfg) == 4 * (2 * w.C + w.C * w.d) + 16 * w.C


def test_vocabulary_shard_needs_tensor_cores(lib):
    w = synthetic.SMALL.replace(C=128, V=4096, d=256)
    assert dg.dg_workspace_bytes(dg.make_config(w, dg.DG_IMPL_SIMT, shard=(0, 1024))) == 0
    assert dg.dg_partials_bytes(dg.make_config(w, dg.DG_IMPL_SIMT)) == 0


def test_vocabulary_shard_takes_e_as_given(lib):
    w = synthetic.SMALL.replace(C=128, V=4096, d=256)
    assert dg.dg_workspace_bytes(dg.make_config(w, dg.DG_IMPL_TC, shard=(0, 1024))) > 0
    w8 = w.replace(e_format=dg.DG_E_FP8)
    assert dg.dg_workspace_bytes(dg.make_config(w8, dg.DG_IMPL_TC)) > 0
    assert dg.dg_workspace_bytes(dg.make_config(w8, dg.DG_IMPL_TC, shard=(0, 1024))) == 0


def test_tensor_core_request_on_unsupported_shape(lib):
    cfg = dg.make_config(synthetic.TINY, dg.DG_IMPL_TC)     # fp32, C=16: not covered
    assert dg.dg_workspace_bytes(cfg) == 0


def test_init_rejects_host_pointers(lib):
    cfg = _cfg()
    buf = (ctypes.c_char * 4096)()
    with pytest.raises(dg.DgError) as e:
        dg.dg_init(cfg, ctypes.addressof(buf), ctypes.addressof(buf), 4096, 0)
    assert e.value.code in (dg.DG_EINVAL, dg.DG_ENOMEM)
    assert dg.dg_last_error(None)


def test_null_context_calls_fail_cleanly(lib):
    assert lib.dg_begin_block(None, 0) == dg.DG_EINVAL
    assert lib.dg_denoise_step(None, None) == dg.DG_EINVAL
    assert lib.dg_read(None, 0, None) == dg.DG_EINVAL
    assert lib.dg_free(None) == dg.DG_OK
    assert lib.dg_inject_stall(None, 0, 0) == dg.DG_EINVAL
    assert lib.dg_self_condition(None, 128, None, None, None, None, None, 0, None) == dg.DG_EINVAL


def test_self_condition_scratch_bytes(lib):
    assert dg.dg_self_condition_scratch_bytes(_cfg(), 256) == 0            # d = 64
    cfg = _cfg(d=1024)
    assert dg.dg_self_condition_scratch_bytes(cfg, 100) == 0               # d_ff % 128 != 0
    n = dg.dg_self_condition_scratch_bytes(cfg, 256)
    assert n >= cfg.C * cfg.d * 2 + cfg.C * 256 * 2 and n % 256 == 0

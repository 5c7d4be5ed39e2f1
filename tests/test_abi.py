"""The C-ABI library loads and exports every entry point ``include/dg.h``
declares; host-side argument checks answer without a device."""
import ctypes
import os
import re

import numpy as np
import pytest

import block_canvas_denoising_b200 as dg
from block_canvas_denoising_b200 import build as dg_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    text = open(os.path.join(ROOT, "include", "dg.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = set(re.findall(r"\b(dg_[a-z_0-9]+)\s*\(", text))
    # typedef'd function pointer types are not exported symbols
    names -= set(re.findall(r"\(\s*\*\s*(dg_[a-z_0-9]+)\s*\)", text))
    return sorted(names)


@pytest.fixture(scope="module")
def libdg():
    dg_build.build()
    return dg.lib()


def test_header_declares_the_boundary():
    names = _declared()
    for required in ("dg_denoise_step", "dg_denoise_loop", "dg_workspace_size", "dg_debug_logits",
                     "dg_error_string", "dg_device_status"):
        assert required in names


def test_library_exports_every_declared_symbol(libdg):
    missing = [n for n in _declared() if not hasattr(libdg, n)]
    assert not missing, missing


def test_default_params_are_serving_defaults(libdg):
    p = libdg.dg_default_params()
    assert (p.tau0, p.tau1, p.max_steps, p.entropy_bound, p.stop_entropy) == (0.8, 0.4, 48, 0.1, 0.005)
    # the struct layout of the binding matches the library's (fields after the
    # seed read back as set by the C side)
    assert (p.seed, p.selection_rule, p.top_k, p.block) == (1234, dg.SELECT_CUMSUM, 1, 0)


def test_selection_rule_checks(libdg):
    # unknown rule, top-k out of [1, 256]: refused on the host
    def call(rule, k):
        prm = dg.Params(selection_rule=rule, top_k=k).c()
        shp = dg._Shape(1, 256, 512, 8192, 0)
        ks = np.zeros(1, np.int32)
        hp = np.zeros(1, np.uint8)
        fake = ctypes.c_void_p(256)
        return libdg.dg_denoise_step(ctypes.byref(shp), ctypes.byref(prm), fake, fake, None,
                                     ks.ctypes.data_as(ctypes.c_void_p), hp.ctypes.data_as(ctypes.c_void_p),
                                     None, *([fake] * 7), fake, ctypes.c_size_t(1 << 30), None)
    assert call(3, 1) == 1
    assert call(-1, 1) == 1
    assert call(dg.SELECT_TOPK, 0) == 1
    assert call(dg.SELECT_TOPK, 257) == 1


def test_error_strings(libdg):
    for code in range(10):
        assert libdg.dg_error_string(code)
    assert libdg.dg_error_string(9) != libdg.dg_error_string(99)


def _call_step(libdg, B=1, L=256, d=512, V=8192, ks=(0,), e_dtype=0, null=False, e_scale=None, params=None):
    shp = dg._Shape(B, L, d, V, e_dtype)
    prm = (params or dg.Params()).c()
    ksa = np.asarray(ks, np.int32)
    hp = np.zeros(max(B, 1), np.uint8)
    fake = ctypes.c_void_p(0 if null else 256)   # never dereferenced: checks fail first
    P = [fake] * 9
    return libdg.dg_denoise_step(ctypes.byref(shp), ctypes.byref(prm), fake, fake, e_scale,
                                 ksa.ctypes.data_as(ctypes.c_void_p), hp.ctypes.data_as(ctypes.c_void_p),
                                 None, *P[:7], fake, ctypes.c_size_t(1 << 30), None)


def test_shape_checks_before_any_device_work(libdg):
    assert _call_step(libdg, L=128) == 2
    assert _call_step(libdg, d=100) == 2
    assert _call_step(libdg, V=1000) == 2
    assert _call_step(libdg, B=0, ks=()) == 2
    assert _call_step(libdg, B=257, ks=[0] * 257) == 2


def test_null_and_range_checks(libdg):
    assert _call_step(libdg, null=True) == 1
    assert _call_step(libdg, ks=(48,)) == 4
    assert _call_step(libdg, ks=(-1,)) == 4


def test_embedder_scale_checks(libdg):
    # the per-row scale is required for the FP8 embedder, refused for bf16,
    # and must be 16-byte aligned (all found before any device work)
    assert _call_step(libdg, e_dtype=1) == 1
    assert _call_step(libdg, e_dtype=0, e_scale=ctypes.c_void_p(512)) == 1
    assert _call_step(libdg, e_dtype=1, e_scale=ctypes.c_void_p(520)) == 1
    assert _call_step(libdg, e_dtype=2, e_scale=ctypes.c_void_p(512)) == 2


def test_workspace_size_zero_for_bad_shape(libdg):
    assert dg.workspace_size(1, 100, 8192) == 0


def test_sharded_entry_points_host_checks(libdg):
    # v_offset must be a multiple of 256; the merge needs at least one shard
    # and record; all refused before any device work
    shp = dg._Shape(1, 256, 512, 4096, 0)
    prm = dg.Params().c()
    ks = np.zeros(1, np.int32)
    hp = np.zeros(1, np.uint8)
    fake = ctypes.c_void_p(256)
    kp = ks.ctypes.data_as(ctypes.c_void_p)
    assert libdg.dg_head_partials(ctypes.byref(shp), ctypes.byref(prm), 100, fake, fake, None, kp, fake, fake,
                                  ctypes.c_size_t(1 << 30), None) == 1
    assert libdg.dg_head_partials(ctypes.byref(shp), ctypes.byref(prm), -256, fake, fake, None, kp, fake, fake,
                                  ctypes.c_size_t(1 << 30), None) == 1
    outs = [fake] * 7
    assert libdg.dg_merge_partials(ctypes.byref(shp), ctypes.byref(prm), fake, 0, 4, kp,
                                   hp.ctypes.data_as(ctypes.c_void_p), None, *outs, fake,
                                   ctypes.c_size_t(1 << 30), None) == 1
    assert libdg.dg_merge_partials(ctypes.byref(shp), ctypes.byref(prm), fake, 2, 0, kp,
                                   hp.ctypes.data_as(ctypes.c_void_p), None, *outs, fake,
                                   ctypes.c_size_t(1 << 30), None) == 1


def test_block_index_checks(libdg):
    # the Philox counter's step word is k | block << 16: a block outside
    # [0, 65535] or more than 65536 steps are refused on the host
    assert _call_step(libdg, params=dg.Params(block=65536)) == 1
    assert _call_step(libdg, params=dg.Params(block=-1)) == 1
    assert _call_step(libdg, params=dg.Params(max_steps=65537)) == 1
    shp = dg._Shape(1, 256, 512, 4096, 0)
    fake = ctypes.c_void_p(256)
    assert libdg.dg_init_canvas(ctypes.byref(shp), ctypes.byref(dg.Params(block=70000).c()), fake, None) == 1
    assert libdg.dg_init_canvas(ctypes.byref(shp), ctypes.byref(dg.Params().c()), None, None) == 1
    bad = dg._Shape(1, 128, 512, 4096, 0)
    assert libdg.dg_init_canvas(ctypes.byref(bad), ctypes.byref(dg.Params().c()), fake, None) == 2
    # the generation: at least one block, a callback, outputs; the last
    # block's index must fit too
    prm = dg.Params().c()
    cb = dg._BLOCK_HIDDEN_FN(lambda *a: 0)
    outs = [fake] * 5
    args = (fake, fake, fake, fake, *outs, fake, ctypes.c_size_t(1 << 30), None)
    assert libdg.dg_generate_blocks(ctypes.byref(shp), ctypes.byref(prm), fake, None, 0, cb, None, fake,
                                    *args) == 1
    steps = np.zeros(4, np.int32)
    sp = steps.ctypes.data_as(ctypes.c_void_p)
    late = dg.Params(block=65534).c()
    assert libdg.dg_generate_blocks(ctypes.byref(shp), ctypes.byref(late), fake, None, 3, cb, None, fake,
                                    fake, sp, fake, fake, *outs, fake, ctypes.c_size_t(1 << 30), None) == 1


def test_device_loop_host_checks(libdg):
    # state size, alignment, step range and null arguments are refused on
    # the host before any device work
    assert libdg.dg_loop_state_bytes(0) == 0 and libdg.dg_loop_state_bytes(257) == 0
    n1 = libdg.dg_loop_state_bytes(1)
    assert n1 >= 256 + 12 and n1 % 256 == 0
    shp = dg._Shape(1, 256, 512, 4096, 0)
    fake = ctypes.c_void_p(4096)
    hp = np.zeros(1, np.uint8)
    st = np.zeros(1, np.int32)
    hpp, stp = hp.ctypes.data_as(ctypes.c_void_p), st.ctypes.data_as(ctypes.c_void_p)

    def call(k_start=0, state=fake, nbytes=n1, hpv=hpp, prm=dg.Params()):
        p = prm.c()
        return libdg.dg_denoise_loop_graph(ctypes.byref(shp), ctypes.byref(p), fake, None, None, k_start, fake,
                                           fake, fake, hpv, stp, fake, fake, fake, fake, fake, state,
                                           ctypes.c_size_t(nbytes), fake, ctypes.c_size_t(1 << 30), None)
    assert call(k_start=48) == 4
    assert call(k_start=-1) == 4
    assert call(state=ctypes.c_void_p(4096 + 16)) == 1     # not 256-byte aligned
    assert call(nbytes=n1 - 1) == 3
    assert call(hpv=None) == 1
    assert call(prm=dg.Params(max_steps=0)) == 1


def test_loop_graph_handle_host_checks(libdg):
    # the reusable device loop refuses bad arguments on the host; without a
    # device it reports DG_ERR_NO_DEVICE and hands back no handle
    n1 = libdg.dg_loop_state_bytes(1)
    shp = dg._Shape(1, 256, 512, 4096, 0)
    fake = ctypes.c_void_p(4096)
    P = ctypes.c_void_p

    def create(state=fake, nbytes=n1, prm=dg.Params(), out=True):
        p = prm.c()
        h = ctypes.c_void_p(1234)
        rc = libdg.dg_loop_graph_create(ctypes.byref(shp), ctypes.byref(p), fake, None, None, fake, fake, fake,
                                        fake, fake, fake, fake, fake, state, ctypes.c_size_t(nbytes), fake,
                                        ctypes.c_size_t(1 << 30), ctypes.byref(h) if out else None)
        return rc, h.value
    assert create(out=False)[0] == 1
    assert create(state=ctypes.c_void_p(4096 + 16)) == (1, None)   # not 256-byte aligned; *out cleared
    assert create(nbytes=n1 - 1) == (3, None)
    assert create(prm=dg.Params(max_steps=0)) == (1, None)
    hp = np.zeros(1, np.uint8)
    st = np.zeros(1, np.int32)
    assert libdg.dg_loop_graph_run(None, 0, hp.ctypes.data_as(P), st.ctypes.data_as(P), None) == 1
    libdg.dg_loop_graph_destroy(None)                                 # a no-op


def test_selfcond_host_checks(libdg):
    # E_t and signal are required and 16-byte aligned; the workspace must
    # hold the signal's scratch (refused before any device work)
    shp = dg._Shape(1, 256, 512, 4096, 0)
    prm = dg.Params().c()
    ks = np.zeros(1, np.int32)
    hp = np.zeros(1, np.uint8)
    fake = ctypes.c_void_p(4096)
    kp, hpp = ks.ctypes.data_as(ctypes.c_void_p), hp.ctypes.data_as(ctypes.c_void_p)

    def call(E_t=fake, signal=fake):
        return libdg.dg_denoise_step_selfcond(ctypes.byref(shp), ctypes.byref(prm), fake, fake, None, E_t, kp, hpp,
                                              *([fake] * 7), signal, fake, ctypes.c_size_t(1 << 40), None)
    assert call(E_t=None) == 1
    assert call(signal=ctypes.c_void_p(4100)) == 1
    assert libdg.dg_embedder_transpose(ctypes.byref(dg._Shape(1, 128, 512, 4096, 0)), fake, fake, None) == 2
    assert libdg.dg_embedder_transpose(ctypes.byref(shp), None, fake, None) == 1
    assert libdg.dg_selfcond_workspace_size(ctypes.byref(dg._Shape(1, 256, 100, 4096, 0))) == 0

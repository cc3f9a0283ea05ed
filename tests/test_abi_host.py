"""The C ABI on the host (no GPU needed): the library loads, exports every
symbol include/moe.h declares, its struct layouts match the header, and its
host-only entry points agree with the oracle.  Device calls here only
exercise argument checks that return before any CUDA work."""
import ctypes as C
import itertools
import os
import re
import subprocess
import tempfile

import numpy as np
import pytest

from mixture_experts_layer_41_b200 import _lib as L
from mixture_experts_layer_41_b200 import api
from mixture_experts_layer_41_b200.inputs import WORKLOADS
from moe_cases import cfg_of
from oracle import moe_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    lib = L.lib()
    names = declared_functions()
    assert len(names) >= 14
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(L.SIGNATURES), set(names) ^ set(L.SIGNATURES)


def test_struct_layout_matches_header():
    src = r"""
#include <stdio.h>
#include <stddef.h>
#include "moe.h"
int main(void) {
  printf("%zu %zu %zu\n", sizeof(moe_config), sizeof(moe_weights), sizeof(moe_stats));
  printf("%zu %zu %zu %zu\n", offsetof(moe_config, routed_scaling), offsetof(moe_config, capacity_factor),
         offsetof(moe_config, shared_intermediate), offsetof(moe_config, aux_alpha));
  return 0;
}
"""
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "t.c")
        exe = os.path.join(d, "t")
        open(c, "w").write(src)
        subprocess.check_call(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), c, "-o", exe])
        out = subprocess.check_output([exe]).decode().split()
    sizes = list(map(int, out))
    assert sizes[:3] == [C.sizeof(L.moe_config), C.sizeof(L.moe_weights), C.sizeof(L.moe_stats)]
    assert sizes[3:] == [L.moe_config.routed_scaling.offset, L.moe_config.capacity_factor.offset,
                         L.moe_config.shared_intermediate.offset, L.moe_config.aux_alpha.offset]


def test_capacity_matches_oracle():
    assert api.moe_capacity(64, 2, 4, 1.25) == 40
    assert api.moe_capacity(8192, 1, 64, 1.0) == 128
    assert api.moe_capacity(4096, 2, 8, 0.0) == -1
    rng = np.random.default_rng(0)
    cfs = [1.0, 1.25, 1.5, 2.0, 1.1, 1.3333334, float(np.float32(1.7))]
    for T, k, E in itertools.product([1, 3, 7, 64, 1000, 4097], [1, 2, 3, 8], [2, 3, 7, 64, 256]):
        if k > E:
            continue
        for cf in cfs + list(rng.uniform(1.0, 3.0, 3).astype(np.float32)):
            cf32 = float(np.float32(cf))
            assert api.moe_capacity(T, k, E, cf32) == O.capacity(T, k, E, cf32), (T, k, E, cf32)


def _cfg(**kw):
    base = dict(num_tokens=64, hidden=64, intermediate=128, num_experts=8, top_k=2)
    base.update(kw)
    return api.make_config(**base)


@pytest.mark.parametrize("kw,status", [
    (dict(), L.MOE_OK),
    (dict(num_experts=1, top_k=1), L.MOE_ERR_INVALID_ARG),
    (dict(top_k=0), L.MOE_ERR_INVALID_TOPK),
    (dict(top_k=9), L.MOE_ERR_INVALID_TOPK),
    (dict(capacity_factor=0.5), L.MOE_ERR_CAPACITY_TOO_TIGHT),
    (dict(capacity_factor=-1.0), L.MOE_ERR_INVALID_ARG),
    (dict(capacity_factor=1.0), L.MOE_OK),
    (dict(aux_alpha=-0.1), L.MOE_ERR_INVALID_ARG),
    (dict(num_tokens=0), L.MOE_ERR_INVALID_ARG),
    (dict(routed_scaling=2.0), L.MOE_ERR_INVALID_ARG),
    (dict(router="sigmoid_group", n_group=4, topk_group=2, routed_scaling=2.5), L.MOE_OK),
    (dict(router="sigmoid_group", n_group=3, topk_group=2, routed_scaling=2.5), L.MOE_ERR_INVALID_ARG),
    (dict(router="sigmoid_group", n_group=8, topk_group=2, routed_scaling=2.5), L.MOE_ERR_INVALID_ARG),
    (dict(router="sigmoid_group", n_group=4, topk_group=5, routed_scaling=2.5), L.MOE_ERR_INVALID_ARG),
    (dict(router="sigmoid_group", n_group=4, topk_group=1, top_k=3, routed_scaling=2.5), L.MOE_ERR_INVALID_TOPK),
    (dict(num_experts=512, top_k=2), L.MOE_ERR_UNSUPPORTED),
    (dict(hidden=60), L.MOE_ERR_UNSUPPORTED),
    (dict(act_dtype="f32", weight_dtype="bf16"), L.MOE_ERR_UNSUPPORTED),
    (dict(act_dtype="f32", weight_dtype="f32", hidden=60, intermediate=30), L.MOE_OK),
    (dict(weight_dtype="q4_affine_g64"), L.MOE_OK),
    (dict(weight_dtype="q4_affine_g64", act="relu"), L.MOE_ERR_UNSUPPORTED),
    (dict(weight_dtype="q4_affine_g64", hidden=96), L.MOE_ERR_UNSUPPORTED),
    (dict(shared_intermediate=64), L.MOE_OK),
    (dict(weight_dtype="q4_affine_g64", shared_intermediate=64), L.MOE_ERR_UNSUPPORTED),
    (dict(weight_layout="fused_gate_up"), L.MOE_OK),
    (dict(weight_layout="fused_gate_up", weight_dtype="q4_affine_g64"), L.MOE_OK),
    (dict(weight_layout="fused_gate_up", act="relu"), L.MOE_ERR_INVALID_ARG),
])
def test_validate(kw, status):
    cfg = _cfg(**kw)
    assert api.moe_validate(cfg) == status
    assert (api.moe_workspace_size(cfg) > 0) == (status == L.MOE_OK)


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_workloads_are_valid(name):
    cfg = cfg_of(WORKLOADS[name])
    assert api.moe_validate(cfg) == L.MOE_OK
    assert api.moe_workspace_size(cfg) > 0


def test_aux_loss_and_health_match_oracle():
    import torch
    rng = np.random.default_rng(3)
    for E, T, k in ((4, 64, 2), (64, 8192, 1), (256, 1000, 8)):
        kept = rng.integers(0, 3 * T * k // E + 1, E).astype(np.int32)
        psum = rng.uniform(0, T / E * 2, E).astype(np.float32)
        cfg = _cfg(num_tokens=T, num_experts=E, top_k=k, aux_alpha=0.01)
        raw, scaled = api.moe_aux_loss(cfg, torch.from_numpy(kept), torch.from_numpy(psum))
        oraw, oscaled = O.aux_loss(kept, psum.astype(np.float64) / T, T, E, float(np.float32(0.01)))
        assert abs(raw - oraw) <= 1e-12 * max(1.0, abs(oraw))
        assert abs(scaled - oscaled) <= 1e-12 * max(1.0, abs(oscaled))
        dropped = int(rng.integers(0, T * k))
        h = api.moe_routing_health(cfg, torch.from_numpy(kept), dropped)
        oh = O.routing_health(kept, dropped, T, k, E)
        for key in ("entropy_ratio", "max_share", "dropped_fraction"):
            assert abs(h[key] - oh[key]) < 1e-12, key
        assert h["collapsed"] == oh["collapsed"]


def test_device_calls_reject_bad_arguments_before_any_launch():
    """Null / misaligned pointers and short workspaces come back as statuses;
    nothing reaches the GPU (this runs on a machine without one)."""
    lib = L.lib()
    cfg = _cfg()
    ws_need = api.moe_workspace_size(cfg)
    fake = 1 << 20   # a 16-byte aligned, never dereferenced address
    st = lib.moe_route(C.byref(cfg), None, fake, None, fake, fake, fake, fake, ws_need, None)
    assert st == L.MOE_ERR_INVALID_ARG
    st = lib.moe_route(C.byref(cfg), fake + 2, fake, None, fake, fake, fake, fake, ws_need, None)
    assert st == L.MOE_ERR_INVALID_ARG
    st = lib.moe_route(C.byref(cfg), fake, fake, None, fake, fake, fake, fake, ws_need - 1, None)
    assert st == L.MOE_ERR_WORKSPACE
    st = lib.moe_route(C.byref(cfg), fake, fake, None, fake, fake, fake, None, ws_need, None)
    assert st == L.MOE_ERR_WORKSPACE
    bad = _cfg(top_k=20)
    st = lib.moe_forward(C.byref(bad), fake, fake, None, None, fake, None, None, None, fake, ws_need, None)
    assert st == L.MOE_ERR_INVALID_TOPK
    w = L.moe_weights()
    st = lib.moe_forward(C.byref(cfg), fake, fake, None, C.byref(w), fake, None, None, None, fake, ws_need, None)
    assert st == L.MOE_ERR_INVALID_ARG
    st = lib.moe_grouped_ffn(C.byref(cfg), fake, fake, None, fake, fake, ws_need, None)
    assert st == L.MOE_ERR_INVALID_ARG
    st = lib.moe_permute(C.byref(cfg), fake, fake, fake, fake, fake, fake, fake, fake, None, fake, ws_need, None)
    assert st == L.MOE_ERR_INVALID_ARG
    st = lib.moe_combine(C.byref(cfg), fake, fake, fake, fake + 8, fake, None)
    assert st == L.MOE_ERR_INVALID_ARG
    cfg_cap = _cfg(capacity_factor=0.9)
    st = lib.moe_combine(C.byref(cfg_cap), fake, fake, fake, None, fake, None)
    assert st == L.MOE_ERR_CAPACITY_TOO_TIGHT
    assert "capacity" in api.moe_status_string(L.MOE_ERR_CAPACITY_TOO_TIGHT)
    # router replay needs the recorded ids; the bias update a finite step >= 0
    st = lib.moe_route_forced(C.byref(cfg), fake, fake, None, None, fake, fake, fake, fake, ws_need, None)
    assert st == L.MOE_ERR_INVALID_ARG
    st = lib.moe_route_forced(C.byref(cfg), fake, fake, None, fake, fake, fake, fake, fake, ws_need - 16, None)
    assert st == L.MOE_ERR_WORKSPACE
    assert lib.moe_update_bias(C.byref(cfg), fake, fake, -1e-3, None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_update_bias(C.byref(cfg), fake, fake, float("inf"), None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_update_bias(C.byref(cfg), None, fake, 1e-3, None) == L.MOE_ERR_INVALID_ARG
    assert lib.moe_update_bias(C.byref(bad), fake, fake, 1e-3, None) == L.MOE_ERR_INVALID_TOPK
    # the fused layout leaves the separate up slots empty
    fused = _cfg(weight_layout="fused_gate_up")
    w = L.moe_weights(w1=fake, w2=fake, w3=fake)
    st = lib.moe_grouped_ffn(C.byref(fused), fake, fake, C.byref(w), fake, fake, ws_need, None)
    assert st == L.MOE_ERR_INVALID_ARG
    bad_layout = _cfg()
    bad_layout.weight_layout = 2
    assert api.moe_validate(bad_layout) == L.MOE_ERR_INVALID_ARG
    bad_gather = _cfg()
    bad_gather.fused_gather = 2
    assert api.moe_validate(bad_gather) == L.MOE_ERR_INVALID_ARG
    # the fused gather drops the expert-sorted copy from the workspace (bf16 experts only)
    assert api.moe_workspace_size(_cfg(fused_gather=True)) < api.moe_workspace_size(_cfg())
    q4 = dict(weight_dtype="q4_affine_g64")
    assert api.moe_workspace_size(_cfg(fused_gather=True, **q4)) == api.moe_workspace_size(_cfg(**q4))


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_workspace_regions(name):
    """moe_workspace_region: the intermediates moe_forward keeps in the
    workspace lie inside it, in order, without overlap, 256-byte aligned,
    with the sizes their shapes give."""
    from mixture_experts_layer_41_b200.inputs import workload
    w = workload(name)
    cfg = cfg_of(w)
    total = api.moe_workspace_size(cfg)
    es = 4 if w.dtype == "f32" else 2
    slots = w.T * w.k
    expect = dict(offsets=4 * (w.E + 1), perm_token=4 * slots, perm_w=4 * slots, slot_row=4 * slots,
                  x_perm=es * slots * w.d, h=es * slots * w.F, y_perm=es * slots * w.d,
                  shared_h=es * w.T * w.shared_F, shared_out=es * w.T * w.d if w.shared_F else 0)
    end = 0
    for region in ("offsets", "perm_token", "perm_w", "slot_row", "x_perm", "h", "y_perm", "shared_h",
                   "shared_out"):
        off, n = api.moe_workspace_region(cfg, region)
        assert off % 256 == 0 and off >= end, (region, off, end)
        assert n == expect[region], (region, n, expect[region])
        end = off + n
        assert end <= total
    # the router's float64 logits partials [ks][T][E] lie before the dispatch buffers
    off, n = api.moe_workspace_region(cfg, "router_logits")
    assert off % 256 == 0 and n % (8 * w.T * w.E) == 0
    assert off + n <= api.moe_workspace_region(cfg, "offsets")[0]
    if w.dtype == "bf16" and w.T >= 512 and (w.router == "sigmoid_group" or w.norm_topk_prob):
        assert n > 0, name          # tensor-core logits live in the workspace
    with pytest.raises(L.MoEError):
        off, n = C.c_size_t(), C.c_size_t()
        L.check(L.lib().moe_workspace_region(C.byref(cfg), L.MOE_WS_REGION_COUNT, C.byref(off), C.byref(n)),
                "region")


@pytest.mark.parametrize("T,d,E,ks", [
    (64, 2048, 128, 16),   # decode-sized: 8 x 4 tiles, four blocks per SM asks 19 slices, capped at 16
    (256, 1024, 64, 8),    # 64 tiles ask 10 slices of 103 elements, rounded up to 128: 8 slices
    (200, 256, 48, 8),     # 25 x 2 tiles ask 12 slices, capped at d / 32 = 8
])
def test_split_router_slice_count(T, d, E, ks):
    """Small batches take the CUDA-core split pass: 8-token x 32-expert tiles
    times as many hidden slices (multiples of 32 elements, at most 16) as give
    148 SMs four blocks each; the workspace holds their float64 partials."""
    cfg = _cfg(num_tokens=T, hidden=d, num_experts=E, top_k=4)
    off, n = api.moe_workspace_region(cfg, "router_logits")
    assert n == ks * T * E * 8, (n // (T * E * 8), ks)


@pytest.mark.parametrize("T,ks", [(16384, 2), (8192, 4), (1024, 4), (512, 9)])
def test_integer_router_slice_count(T, ks):
    """The integer tensor-core plan (bf16, T >= 512) splits the hidden
    dimension (112 K-blocks of 64 at d = 7168) into the slice count whose
    rounds of 148 CTAs times K-blocks per CTA, plus four K-blocks of fixed
    cost, are fewest; the workspace holds the float64 partials."""
    cfg = _cfg(num_tokens=T, hidden=7168, num_experts=256, top_k=8, router="sigmoid_group", n_group=8,
               topk_group=4, routed_scaling=2.5)
    off, n = api.moe_workspace_region(cfg, "router_logits")
    assert n == ks * T * 256 * 8, (n // (T * 256 * 8), ks)


def _router_plan_sizes(env_extra):
    """Workspace size and router-logits region of two bf16 configurations,
    in a fresh process (the router switch is read once per process)."""
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = (
        "import sys; sys.path.insert(0, %r)\n"
        "from mixture_experts_layer_41_b200 import api\n"
        "for T, d, E, k, kw in [(1024, 1024, 256, 8, dict(router='sigmoid_group', n_group=8, topk_group=4)),\n"
        "                       (600, 512, 8, 2, {})]:\n"
        "    cfg = api.make_config(num_tokens=T, hidden=d, intermediate=64, num_experts=E, top_k=k, **kw)\n"
        "    print(api.moe_workspace_size(cfg), api.moe_workspace_region(cfg, 'router_logits')[1])\n" % root)
    env = {k: v for k, v in os.environ.items() if k != "MOE_ROUTER_TC"}
    env.update(env_extra)
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    return [tuple(int(v) for v in line.split()) for line in r.stdout.split("\n") if line.strip()]


def test_bf16_router_switch_changes_the_plan():
    """MOE_ROUTER_TC=bf16 puts bf16 batches of 512 tokens or more on the bf16
    selection-grade tensor-core logits instead of the integer ones: the
    workspace the plan sizes differs (its own weight slices and slice count)."""
    default = _router_plan_sizes({})
    bf16 = _router_plan_sizes({"MOE_ROUTER_TC": "bf16"})
    assert len(default) == len(bf16) == 2
    assert all(a[0] != b[0] for a, b in zip(default, bf16))

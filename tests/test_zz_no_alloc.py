"""moe_route_noalloc: the router for callers that may not allocate device
memory (no cudaMalloc, no workspace; e.g. code inside a framework plugin that
owns all device memory, or a serving loop that forbids allocation after
start-up).  Its score scratch is a fixed array inside the library.  Checked
through the C ABI against moe_route on the same inputs, bit for bit (routing
is compared exactly everywhere in this suite), on two calls in a row; and the
size limit is enforced before anything is enqueued.

Kept in a file that sorts last so that a run stopping at its first failure
has already run every other test."""
import numpy as np
import pytest
import torch

import sparse_moe_transformer_fwd_b200 as moe
from moe_inputs import CONFIGS, make_x, make_router

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0") if torch.cuda.is_available() else None


def _route_both(cfg, seed):
    x = make_x(cfg, seed, "cpu").to(DEV)
    w, b = make_router(cfg, seed, "cpu")
    w, b = w.to(DEV), b.to(DEV)
    shape = moe.make_shape(cfg.T, cfg.d_model, cfg.n_experts, cfg.top_k, cfg.d_expert,
                           cfg.n_shared, cfg.routed_scale, cfg.precision)
    ws = moe.alloc_workspace(shape, DEV)
    idx_ref = torch.empty(cfg.T, cfg.top_k, dtype=torch.int32, device=DEV)
    g_ref = torch.empty(cfg.T, cfg.top_k, dtype=torch.float32, device=DEV)
    moe.moe_route(shape, x, w, b, idx_ref, g_ref, ws)
    assert moe.moe_check_status(ws) == 0
    outs = []
    for _ in range(2):  # two calls in a row share the fixed scratch
        idx = torch.full((cfg.T, cfg.top_k), -1, dtype=torch.int32, device=DEV)
        g = torch.full((cfg.T, cfg.top_k), -1.0, dtype=torch.float32, device=DEV)
        moe.moe_route_noalloc(shape, x, w, b, idx, g)
        torch.cuda.synchronize()
        outs.append((idx.cpu(), g.cpu()))
    return (idx_ref.cpu(), g_ref.cpu()), outs


# T=64: the small-batch router; T=600: 32-token tiles; T=4096: 64-token tiles
@pytest.mark.parametrize("name,T", [("decode", 64), ("tiny", 128), ("decode", 600),
                                    ("decode", 4096)])
def test_noalloc_route_matches_moe_route(name, T):
    cfg = CONFIGS[name].with_(T=T)
    (idx_ref, g_ref), outs = _route_both(cfg, seed=5)
    for idx, g in outs:
        assert torch.equal(idx, idx_ref)
        assert np.array_equal(g.numpy().view(np.uint32), g_ref.numpy().view(np.uint32))


def test_noalloc_route_rejects_oversize():
    cfg = CONFIGS["decode"].with_(T=moe.MOE_ROUTE_NOALLOC_MAX_SCORES // 256 + 1)
    shape = moe.make_shape(cfg.T, cfg.d_model, cfg.n_experts, cfg.top_k, cfg.d_expert)
    t = torch.empty(16, dtype=torch.int32, device=DEV)
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_route_noalloc(shape, t.view(torch.bfloat16), t.view(torch.bfloat16),
                              t.float(), t, t.float())
    assert ei.value.code == moe._native.MOE_ERR_INVALID_ARG
    assert "exceeds" in moe.moe_last_error()


_RESET_CHILD = r"""
import ctypes, sys
import numpy as np
sys.path.insert(0, sys.argv[1])
import sparse_moe_transformer_fwd_b200 as moe
rt = ctypes.CDLL(sys.argv[2])
vp, sz = ctypes.c_void_p, ctypes.c_size_t
rt.cudaMalloc.argtypes = [ctypes.POINTER(vp), sz]
rt.cudaMemcpy.argtypes = [vp, vp, sz, ctypes.c_int]
rt.cudaFree.argtypes = [vp]
T, d, E, k = 600, 7168, 256, 8
rng = np.random.default_rng(7)
bf = lambda a: (a.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
x = bf(rng.standard_normal((T, d)))
w = bf(rng.standard_normal((E, d)) * 0.006)
b = (rng.random(E) * 0.2 - 0.1).astype(np.float32)
shape = moe.make_shape(T, d, E, k, 2048)
L = moe.lib()

def dev(a):
    p = vp()
    assert rt.cudaMalloc(ctypes.byref(p), a.nbytes) == 0
    assert rt.cudaMemcpy(p, a.ctypes.data, a.nbytes, 1) == 0
    return p

def route(noalloc):
    xp, wp, bp = dev(x), dev(w), dev(b)
    idx, g = np.zeros((T, k), np.int32), np.zeros((T, k), np.float32)
    ip, gp = dev(idx), dev(g)
    if noalloc:
        rc = L.moe_route_noalloc(ctypes.byref(shape), xp, wp, bp, ip, gp, None)
    else:
        n = L.moe_workspace_size(ctypes.byref(shape))
        ws = dev(np.zeros(n, np.uint8))
        rc = L.moe_route(ctypes.byref(shape), xp, wp, bp, ip, gp, ws, n, None)
    assert rc == 0, L.moe_last_error()
    assert rt.cudaMemcpy(idx.ctypes.data, ip, idx.nbytes, 2) == 0
    assert rt.cudaMemcpy(g.ctypes.data, gp, g.nbytes, 2) == 0
    for p in (xp, wp, bp, ip, gp):
        rt.cudaFree(p)
    return idx, g

def same(a, b):
    return np.array_equal(a[0], b[0]) and np.array_equal(a[1].view(np.uint32), b[1].view(np.uint32))

ref = route(False)
first = route(True)
assert same(first, ref), "before the reset"
assert rt.cudaDeviceReset() == 0          # ends this process's context only
after = route(True)                       # a new context: the scratch is looked up again
assert same(after, ref), "no-alloc router after the reset"
assert same(route(False), ref), "workspace router after the reset"
print("reset ok")
"""


def test_noalloc_route_after_device_reset():
    """A process that resets its device (cudaDeviceReset) and routes again gets
    the same bits as before: the library looks the scratch address up again
    in the new context (whose handle may equal the old one; its id does not),
    and re-applies its kernel attributes.  Run in a child process, which owns
    the only context it resets; buffers come from the CUDA runtime directly."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    cudart = next(p for p in ("/usr/local/cuda/lib64/libcudart.so.12",
                              "/usr/local/cuda/lib64/libcudart.so") if os.path.exists(p))
    r = subprocess.run([sys.executable, "-c", _RESET_CHILD, root, cudart], capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0 and "reset ok" in r.stdout, r.stdout + r.stderr

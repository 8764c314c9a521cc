"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point include/gmm_b200.h declares, and rejects invalid arguments
on the host before launching anything."""
import ctypes
import os
import re
import subprocess

import pytest

from means_clustering_gmm_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = []
    inc = os.path.join(ROOT, "include")
    for f in sorted(os.listdir(inc)):
        if not f.endswith(".h"):
            continue
        src = open(os.path.join(inc, f)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^[A-Za-z_][\w \*]*?\b([a-z_][a-z0-9_]*)\s*\(", src, flags=re.M):
            if not m.group(0).lstrip().startswith(("#", "typedef", "return")):
                names.append(m.group(1))
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = _declared_functions()
    for n in ["gmm_em_step", "gmm_finalize", "kmeans_step", "gmm_workspace_size",
              "kmeans_workspace_size", "gmm_last_error", "gmm_workspace_init", "gmm_fit",
              "gmm_init_kmeans"]:
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = _lib.load()
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    for n in _declared_functions():
        assert n in exported, n
        assert getattr(lib, n) is not None
        assert n in _lib.SIGNATURES, n


@pytest.mark.gpu
def test_kernels_run_sm100_code():
    """The device code the library runs reports binary version 100 (sm_100a);
    asked at run time through cudaFuncGetAttributes on one of its kernels."""
    import torch
    torch.cuda.init()
    assert _lib.load().gmm_device_binary_version() == 100


def test_build_targets_sm100a_only():
    """The build compiles for sm_100a and nothing else."""
    from means_clustering_gmm_b200 import build
    assert build.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]


def test_workspace_sizes():
    lib = _lib.load()
    assert lib.gmm_workspace_size(0, 16, 8, 0) == 0
    assert lib.gmm_workspace_size(100, 0, 8, 0) == 0
    assert lib.gmm_workspace_size(100, 16, 0, 0) == 0
    assert lib.gmm_workspace_size(100, 2000, 8, 0) == 0
    assert lib.gmm_workspace_size(100, 16, 8, 7) == 0
    small = lib.gmm_workspace_size(4096, 16, 8, 0)
    big = lib.gmm_workspace_size(1_000_000, 128, 256, 0)
    assert 0 < small < big
    assert lib.kmeans_workspace_size(32, 65536, 128, 1024) > 0
    assert lib.kmeans_workspace_size(0, 10, 4, 4) == 0
    assert lib.kmeans_workspace_size(1, 10, 4, 5000) == 0


def _direct_slots(K):
    want = K // 8 if K > 2048 else max(K // 16, 64)
    return min(K, min(want, 512))


def _block_budget(N, d):
    """Bytes the direct-form score block may take: X at 16 bits per
    element, clamped to [512 MiB, 4 GiB]."""
    return min(max(N * d * 2, 512 << 20), 4 << 30)


def test_workspace_holds_one_chunk_of_direct_form_scores():
    """The tensor-core path keeps the fp32 direct-form scores of one point
    chunk at a time ([slots x chunk], slots = 64 up to K = 1024, K/16 up to
    K = 2048, K/8 above, at most 512), at most the size of X at 16 bits per
    element (clamped to [512 MiB, 4 GiB]).  So the workspace never grows
    past 4 GiB of scores plus the per-point l_n (4 bytes a point, and one
    fp64 per 128-point tile) and the fixed parts, and at N = 10^7, d = 128,
    K = 4096 (bf16, 2.56 GB of X) it is smaller than X."""
    lib = _lib.load()
    BF16 = _lib.GMM_BF16
    for K in (256, 2048, 4096):
        fixed = 148 * K * (1 + 2 * 128) * 8 + (64 << 20)   # partial rows, image, small parts
        for N in (20_000_000, 40_000_000, 80_000_000):
            ws = lib.gmm_workspace_size(N, 128, K, BF16)
            assert 0 < ws <= (4 << 30) + N * (4 + 8 / 128) + fixed, (K, N, ws)
    x_bytes = 10_000_000 * 128 * 2
    assert lib.gmm_workspace_size(10_000_000, 128, 4096, BF16) < x_bytes
    # while the block fits its budget the whole of N is one chunk, and the
    # block grows with N
    for K in (256, 2048, 4096):
        a = lib.gmm_workspace_size(50_000, 128, K, BF16)
        b = lib.gmm_workspace_size(200_000, 128, K, BF16)
        assert b - a >= _direct_slots(K) * 4 * 150_000, (K, a, b)


def test_point_chunks():
    """gmm_point_chunk: N when the call runs in one piece (always on the
    CUDA-core kernels, and on the tensor cores while the direct-form block
    of all N points fits its budget); otherwise equal chunks of whole waves
    of 128-point tiles (148 of them) whose block fits.  gmm_set_point_chunk
    caps it (rounded up to 128 points) and never raises it past what the
    workspace was sized for."""
    lib = _lib.load()
    F32, BF16 = _lib.GMM_F32, _lib.GMM_BF16
    wave = 128 * 148
    assert lib.gmm_point_chunk(1_000_000, 128, 256, F32, 0) == 1_000_000
    assert lib.gmm_point_chunk(16_777_216, 32, 16, BF16, 0) == 16_777_216
    assert lib.gmm_point_chunk(4096, 16, 8, F32, 0) == 4096          # CUDA-core kernels
    assert lib.gmm_point_chunk(100_000_000, 64, 40, F32, 2) == 100_000_000   # forced CUDA core
    assert lib.gmm_point_chunk(0, 128, 256, F32, 0) == -1
    for N, d, K in [(10_000_000, 128, 4096), (3_000_000, 128, 2048), (50_000_000, 128, 2048),
                    (200_000_000, 32, 16), (60_000_000, 32, 256), (100_000_000, 64, 200)]:
        slots = _direct_slots(K)
        budget = _block_budget(N, d)
        c = lib.gmm_point_chunk(N, d, K, BF16, 0)
        if slots * 4 * N <= budget:
            assert c == N, (N, d, K, c)
            continue
        assert c % wave == 0 and 0 < c < N, (N, d, K, c)
        assert slots * 4 * c <= budget, (N, d, K, c)
        n_chunks = -(-N // c)
        assert c - (-(-N // n_chunks)) < wave, (N, d, K, c)   # equal chunks
    assert lib.gmm_point_chunk(10_000_000, 128, 4096, BF16, 0) == 1_117_696
    try:
        assert lib.gmm_set_point_chunk(50_000) == 0
        assert lib.gmm_point_chunk(1_000_000, 128, 256, F32, 0) == 50_048
        assert lib.gmm_point_chunk(1_000_000, 128, 256, F32, 2) == 1_000_000
        assert lib.gmm_point_chunk(10_000_000, 128, 4096, BF16, 0) == 50_048
        assert lib.gmm_set_point_chunk(1 << 40) == 0
        assert lib.gmm_point_chunk(10_000_000, 128, 4096, BF16, 0) == 1_117_696
        assert lib.gmm_set_point_chunk(-1) == _lib.GMM_ERR_INVALID_ARG
    finally:
        assert lib.gmm_set_point_chunk(0) == 0
    assert lib.gmm_point_chunk(1_000_000, 128, 256, F32, 0) == 1_000_000


def test_collecting_timer_host_side():
    """The collecting kernel timer's host bookkeeping: end without begin is
    rejected, a begin/end pair with no launch in between reports no region
    (no CUDA call is made)."""
    lib = _lib.load()
    n = ctypes.c_int64(-1)
    assert lib.gmm_kernel_timer_end(None, 0, ctypes.byref(n)) == _lib.GMM_ERR_INVALID_ARG
    assert lib.gmm_kernel_timer_begin() == 0
    assert lib.gmm_kernel_timer_end(None, 1, ctypes.byref(n)) == _lib.GMM_ERR_INVALID_ARG
    assert lib.gmm_kernel_timer_begin() == 0
    assert lib.gmm_kernel_timer_end(None, 0, ctypes.byref(n)) == 0
    assert n.value == 0


def test_invalid_arguments_rejected_before_launch():
    """Null pointers, bad sizes, misalignment and a short workspace return
    GMM_ERR_INVALID_ARG on the host (no CUDA call is made, so this runs
    without a GPU)."""
    lib = _lib.load()
    A = 1 << 20  # a fake, 256-aligned, never-dereferenced address
    ws = lib.gmm_workspace_size(100, 4, 3, 0)
    ok = dict(X=A, dt=0, N=100, d=4, K=3, m=A, v=A, w=A, st=A, ll=None, lt=None, ws=A,
              wsb=ws, fl=0, s=None)

    def call(**kw):
        a = dict(ok, **kw)
        return lib.gmm_em_step(a["X"], a["dt"], a["N"], a["d"], a["K"], a["m"], a["v"], a["w"],
                               a["st"], a["ll"], a["lt"], a["ws"], a["wsb"], a["fl"], a["s"])

    E = _lib.GMM_ERR_INVALID_ARG
    assert call(X=None) == E
    assert call(m=None) == E
    assert call(st=None) == E
    assert call(ws=None) == E
    assert call(N=0) == E
    assert call(d=0) == E
    assert call(K=0) == E
    assert call(d=5000) == E
    assert call(dt=9) == E
    assert call(X=A + 4) == E          # X must be 16-byte aligned
    assert call(ws=A + 64) == E        # workspace must be 256-byte aligned
    assert call(wsb=ws - 1) == E       # workspace too small
    assert call(fl=64) == E            # unknown flag
    # the test-only stall flag needs the one-CTA tensor-core kernel
    U = _lib.GMM_ERR_UNSUPPORTED
    wsb = lib.gmm_workspace_size(1000, 64, 200, 0)
    assert call(N=1000, d=64, K=200, wsb=wsb, fl=_lib.GMM_FLAG_TEST_STALL) == U
    assert call(N=1000, d=64, K=20, wsb=wsb, fl=_lib.GMM_FLAG_TEST_STALL | 2) == U
    assert call(N=1000, d=16, K=20, wsb=wsb, fl=_lib.GMM_FLAG_TEST_STALL) == U
    assert lib.gmm_finalize(A, 100, 4, 3, ctypes.c_float(0.0), A, A, A, A, 4096, None) == E
    assert lib.gmm_finalize(None, 100, 4, 3, ctypes.c_float(1e-6), A, A, A, A, 4096, None) == E
    kws = lib.kmeans_workspace_size(2, 100, 4, 3)
    km = lambda **kw: lib.kmeans_step(kw.get("X", A), 0, kw.get("B", 2), 100, 4,
                                      kw.get("K", 3), kw.get("C", A), A, kw.get("nC", A + 256),
                                      None, None, A, kw.get("wsb", kws), 0, None)
    assert km(X=None) == E
    assert km(B=0) == E
    assert km(K=5000) == E
    assert km(nC=A) == E               # output may not alias the input centroids
    assert km(wsb=kws - 1) == E
    assert lib.gmm_workspace_init(None, 256, None) == E
    assert lib.gmm_last_error(None, None) == E


def test_fit_and_init_reject_invalid_arguments_before_launch():
    """gmm_fit / gmm_init_kmeans check their arguments on the host (no CUDA
    call is made on these paths, so this runs without a GPU)."""
    lib = _lib.load()
    A = 1 << 20
    E = _lib.GMM_ERR_INVALID_ARG
    N, d, K = 100, 4, 3
    fws = lib.gmm_fit_workspace_size(N, d, K, 0)
    assert fws > lib.gmm_workspace_size(N, d, K, 0) > 0
    assert lib.gmm_fit_workspace_size(0, d, K, 0) == 0

    def fit(**kw):
        a = dict(X=A, N=N, it=10, tol=1e-6, vf=1e-6, tr=None, info=None, ws=A, wsb=fws, fl=0)
        a.update(kw)
        return lib.gmm_fit(a["X"], 0, a["N"], d, K, A, A, A, a["it"], a["tol"],
                           ctypes.c_float(a["vf"]), a["tr"], a["info"], a["ws"], a["wsb"],
                           a["fl"], None)

    assert fit(it=0) == E
    assert fit(tol=-1.0) == E
    assert fit(vf=0.0) == E
    assert fit(wsb=fws - 1) == E
    assert fit(X=None) == E
    assert fit(N=0) == E
    assert fit(tr=A + 4) == E          # trace must be 8-byte aligned
    assert fit(info=A + 2) == E        # info must be 4-byte aligned
    assert fit(fl=64) == E
    iws = lib.gmm_init_kmeans_workspace_size(N, d, K)
    assert iws > lib.kmeans_workspace_size(1, N, d, K) > 0
    assert lib.gmm_init_kmeans_workspace_size(N, d, 5000) == 0

    def init(**kw):
        a = dict(X=A, it=3, vf=1e-6, ws=A, wsb=iws, m=A)
        a.update(kw)
        return lib.gmm_init_kmeans(a["X"], 0, N, d, K, a["it"], ctypes.c_float(a["vf"]), a["m"],
                                   A, A, None, a["ws"], a["wsb"], None)

    assert init(it=0) == E
    assert init(vf=-1.0) == E
    assert init(wsb=iws - 1) == E
    assert init(X=A + 8) == E
    assert init(m=None) == E


def test_batched_sizes_and_checks():
    lib = _lib.load()
    one = lib.gmm_workspace_size(5000, 64, 40, 0)
    four = lib.gmm_batched_workspace_size(4, 5000, 64, 40, 0)
    assert four >= 4 * one and lib.gmm_batched_workspace_size(0, 5000, 64, 40, 0) == 0
    A = 1 << 20
    E = _lib.GMM_ERR_INVALID_ARG
    call = lambda **kw: lib.gmm_em_step_batched(
        kw.get("X", A), 0, kw.get("B", 4), kw.get("N", 5000), 64, 40, A, A, A, A, None, None, A,
        kw.get("wsb", four), 0, None)
    assert call(wsb=four - 1) == E
    assert call(B=0) == E
    assert call(X=None) == E
    # 5001 x 64 fp32 rows are 16-byte aligned, 4097 x 3 bf16 per problem are not
    assert lib.gmm_em_step_batched(A, 1, 2, 4097, 3, 4, A, A, A, A, None, None, A,
                                   lib.gmm_batched_workspace_size(2, 4097, 3, 4, 1), 0,
                                   None) == E
    assert lib.gmm_finalize_batched(A, 2, 100, 4, 3, ctypes.c_float(0.0), A, A, A, A, 4096,
                                    None) == E


def test_soft_assign_rejects_invalid_arguments():
    lib = _lib.load()
    A = 1 << 20
    E = _lib.GMM_ERR_INVALID_ARG
    wsb = lib.gmm_workspace_size(100, 4, 3, 0)
    call = lambda **kw: lib.gmm_soft_assign(A, 0, 100, 4, 3, A, A, A, kw.get("r", 2),
                                            ctypes.c_float(kw.get("tau", 0.1)), kw.get("ids", A),
                                            A, None, A, kw.get("wsb", wsb), kw.get("fl", 0), None)
    assert call(r=0) == E
    assert call(r=9) == E
    assert call(tau=-0.1) == E
    assert call(tau=1.5) == E
    assert call(ids=None) == E
    assert call(wsb=wsb - 1) == E
    assert call(fl=1) == E


def test_status_strings():
    assert _lib.status_string(0) == "GMM_OK"
    assert _lib.status_string(6) == "GMM_ERR_RANGE"
    assert _lib.status_string(99) == "GMM_ERR_UNKNOWN"


def test_binding_chunk_and_timer_helpers_host_side():
    """The binding's point_chunk / set_point_chunk / KernelTimer marshal the
    host-only calls (no CUDA call is made here)."""
    import torch
    import means_clustering_gmm_b200 as gmm
    assert gmm.point_chunk(1_000_000, 128, 256) == 1_000_000
    assert gmm.point_chunk(10_000_000, 128, 4096, torch.bfloat16) == 1_117_696
    with pytest.raises(ValueError):
        gmm.point_chunk(0, 128, 256)
    try:
        gmm.set_point_chunk(1000)
        assert gmm.point_chunk(1_000_000, 128, 256) == 1024
    finally:
        gmm.set_point_chunk(0)
    with pytest.raises(gmm.GmmError):
        gmm.set_point_chunk(-5)
    with gmm.KernelTimer() as t:
        pass
    assert t.ms == []

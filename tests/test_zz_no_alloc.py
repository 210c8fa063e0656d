"""awq_search_noalloc — the search for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc: a plugin inside a framework that owns every byte
of device memory, a process whose memory budget was fixed at start-up, or a loop that
must not risk an allocation's synchronisation or failure. For them the library runs the
search in one fixed array compiled into the library instead of pooled work space. These
tests call that entry point through the C ABI and compare it with awq_search_ex on the
same inputs bit for bit, on two calls in a row (the array keeps the previous call's
contents, so the second call must not be affected by the first); they check that layers
beyond the array are refused and that the calls allocate no device memory. This file is
collected last on purpose.
"""
import ctypes

import pytest
import torch

import post_quantization_column_b200 as awq
from workloads import custom_spec, generate, WORKLOADS

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 64 << 20   # AWQ_NOALLOC_SCRATCH_BYTES in include/awq_search.h


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = awq.library()
    lib.awq_search_noalloc.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int64,
                                       ctypes.c_int64, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                       ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    lib.awq_search_noalloc.restype = ctypes.c_int
    return lib


def _outputs(K, N, group, n_grid):
    dev = torch.device("cuda")
    return (torch.empty(K, dtype=torch.float32, device=dev),
            torch.empty(K, N // 8, dtype=torch.int32, device=dev),
            torch.empty(K // group, N, dtype=torch.float16, device=dev),
            torch.empty(K // group, N, dtype=torch.float16, device=dev),
            torch.empty(n_grid, dtype=torch.float32, device=dev),
            torch.full((1,), -1, dtype=torch.int32, device=dev))


def _noalloc(lib, X, W, group, n_grid, outs):
    M, K = X.shape
    N = W.shape[1]
    dtype = 0 if X.dtype == torch.bfloat16 else 1
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.awq_search_noalloc(p(X), p(W), dtype, M, K, N, group, n_grid, p(outs[0]), p(outs[1]), p(outs[2]),
                                  p(outs[3]), p(outs[4]), p(outs[5]), stream)


def _same(ref, outs):
    # the same launch sequence on the same inputs: every output bit for bit, losses included
    for name, got in zip(("scales", "codes", "steps", "zeros", "losses", "best_index"), outs):
        assert torch.equal(getattr(ref, name), got), name


def test_two_calls_in_a_row_match_the_pooled_entry_point(lib):
    layers = [custom_spec(300, 384, 520, seed=21), custom_spec(256, 512, 768, law="abs_normal", sigma=1.0,
                                                              outlier_mult=50.0, seed=22)]
    for spec in layers:   # the second layer runs on the array the first one left behind
        X, W = (t.cuda() for t in generate(spec))
        ref = awq.search(X, W, spec.group, spec.n_grid)
        outs = _outputs(spec.K, spec.N, spec.group, spec.n_grid)
        st = _noalloc(lib, X, W, spec.group, spec.n_grid, outs)
        assert st == 0, lib.awq_last_error_message()
        torch.cuda.synchronize()
        _same(ref, outs)


def test_fp32_layer_and_repeat_on_the_same_inputs(lib):
    spec = WORKLOADS["single_linear_128x256x256_f32"]
    X, W = (t.cuda() for t in generate(spec))
    ref = awq.search(X, W, spec.group, spec.n_grid)
    for _ in range(2):
        outs = _outputs(spec.K, spec.N, spec.group, spec.n_grid)
        assert _noalloc(lib, X, W, spec.group, spec.n_grid, outs) == 0, lib.awq_last_error_message()
        torch.cuda.synchronize()
        _same(ref, outs)


def test_calls_allocate_no_device_memory(lib):
    spec = custom_spec(256, 384, 512, seed=23)
    X, W = (t.cuda() for t in generate(spec))
    outs = _outputs(spec.K, spec.N, spec.group, spec.n_grid)
    assert _noalloc(lib, X, W, spec.group, spec.n_grid, outs) == 0   # first call: the array and its address
    torch.cuda.synchronize()
    # give back what the library's pool and torch's cache hold, so that an allocation
    # from either would have to take new device memory and show in the free count
    awq.release_cached()
    torch.cuda.empty_cache()
    free_before, _ = torch.cuda.mem_get_info()
    for _ in range(2):
        assert _noalloc(lib, X, W, spec.group, spec.n_grid, outs) == 0
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    assert free_after == free_before


def test_layers_beyond_the_array_are_refused(lib):
    M, K, N, group, n_grid = 4096, 4096, 4096, 128, 20      # needs ~0.85 GB of work space
    X = torch.zeros(M, K, dtype=torch.bfloat16, device="cuda")
    W = torch.zeros(K, N, dtype=torch.bfloat16, device="cuda")
    outs = _outputs(K, N, group, n_grid)
    st = _noalloc(lib, X, W, group, n_grid, outs)
    assert st == 2
    msg = lib.awq_last_error_message().decode()
    assert "work space" in msg and str(SCRATCH_BYTES) in msg


def test_fp32_layer_refused_when_only_its_bf16_copy_of_X_overflows(lib):
    # the bf16 layer fits the array; its fp32 form also needs M*K*2 bytes for the bf16
    # copy of X, which pushes it past the array
    M, K, N, group, n_grid = 16384, 1024, 512, 128, 20
    assert awq.workspace_bytes(M, K, N, group, n_grid, torch.bfloat16) <= SCRATCH_BYTES
    assert awq.workspace_bytes(M, K, N, group, n_grid, torch.float32) > SCRATCH_BYTES
    X = torch.zeros(M, K, dtype=torch.float32, device="cuda")
    W = torch.zeros(K, N, dtype=torch.float32, device="cuda")
    outs = _outputs(K, N, group, n_grid)
    assert _noalloc(lib, X, W, group, n_grid, outs) == 2
    assert str(awq.workspace_bytes(M, K, N, group, n_grid, torch.float32)) in lib.awq_last_error_message().decode()

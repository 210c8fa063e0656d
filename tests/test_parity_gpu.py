"""CUDA search vs the CPU oracle, element by element (B200 only).

Small layers use the complete oracle; they span several 128 x 256 output tiles,
ragged row/column tails, ragged K blocks (group 32 with K not a multiple of 64),
every group size and a few grid sizes.
"""
import numpy as np
import pytest
import torch

import oracle as O
import post_quantization_column_b200 as awq
from tests import parity as P
from workloads import WORKLOADS, custom_spec, generate, as_f32_numpy

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


def test_single_linear_layer_fp32():
    spec = WORKLOADS["single_linear_128x256x256_f32"]
    X, W = generate(spec)
    P.full_parity(X, W, spec.group, spec.n_grid)


@pytest.mark.parametrize("M,K,N,group,n_grid,law,dtype", [
    (300, 384, 520, 128, 20, "normal", "bf16"),      # ragged M and N tails, 3 x 3 tiles
    (200, 160, 264, 32, 20, "normal", "bf16"),       # group 32, K = 2.5 K-blocks
    (129, 320, 776, 64, 7, "abs_normal", "bf16"),    # group 64, one extra row, odd grid
    (64, 256, 256, 128, 1, "normal", "bf16"),        # a single candidate
    (260, 512, 1032, 128, 20, "abs_normal", "f32"),  # fp32 inputs, ragged tails
    (1, 128, 8, 128, 20, "normal", "bf16"),          # one token, one packed word
    (96, 256, 264, 128, 64, "normal", "bf16"),       # the largest grid (64 candidates)
    (64, 160, 136, 32, 64, "abs_normal", "bf16"),    # largest grid with group 32
])
def test_small_layers(M, K, N, group, n_grid, law, dtype):
    spec = custom_spec(M, K, N, dtype=dtype, law=law, group=group, n_grid=n_grid, seed=M + K + N,
                       sigma=1.0 if law == "abs_normal" else 0.5,
                       outlier_mult=50.0 if law == "abs_normal" else 20.0)
    X, W = generate(spec)
    P.full_parity(X, W, group, n_grid)


@pytest.mark.parametrize("variant", ["1", "2"])
@pytest.mark.parametrize("M,K,N,group,dtype", [(300, 384, 520, 128, "bf16"), (129, 320, 776, 64, "f32"),
                                               (520, 256, 264, 32, "bf16")])
def test_both_gemm_variants(M, K, N, group, dtype, variant, monkeypatch):
    # the one-SM (128 x 256 tiles) and two-SM (256 x 256 tiles, cta_group::2) loss
    # GEMMs, including odd row-tile counts that leave half of the last pair empty
    monkeypatch.setenv("AWQ_GEMM_VARIANT", variant)
    spec = custom_spec(M, K, N, dtype=dtype, group=group, seed=M * 7 + N)
    X, W = generate(spec)
    P.full_parity(X, W, group, 20)


@pytest.mark.parametrize("M,K,N,group,n_grid,dtype", [(300, 384, 520, 128, 20, "bf16"), (129, 320, 776, 64, 7, "f32"),
                                                      (520, 256, 264, 32, 20, "bf16"), (64, 160, 136, 32, 64, "bf16")])
def test_reference_launch_forms(M, K, N, group, n_grid, dtype, monkeypatch):
    # The one-SM GEMM scores the candidates either in one launch with the reference tiles
    # (Y within L2) or after a reference launch, walking every candidate of a column tile
    # before the next (Y larger than L2); the environment forces each form at this size.
    # Both match the oracle, and each tile's squared error is the same bits in both.
    spec = custom_spec(M, K, N, dtype=dtype, group=group, n_grid=n_grid, seed=M * 3 + K + N)
    X, W = generate(spec)
    monkeypatch.setenv("AWQ_QDQ", "standalone")
    outs = {}
    for form in ("fused", "own"):
        monkeypatch.setenv("AWQ_REFERENCE_LAUNCH", form)
        P.full_parity(X, W, group, n_grid)
        outs[form] = awq.search(X.cuda(), W.cuda(), group, n_grid, tile_sq_err=True)
    for name in ("scales", "codes", "steps", "zeros", "losses", "best_index", "tile_sq_err"):
        assert torch.equal(getattr(outs["fused"], name), getattr(outs["own"], name)), name


@pytest.mark.parametrize("M,K,N,n_grid,quantizer", [(300, 384, 520, 20, "asym"), (129, 256, 776, 64, "asym"),
                                                     (520, 512, 264, 11, "sym"), (1, 128, 8, 20, "asym"),
                                                     (1000, 1024, 2056, 20, "asym"), (64, 256, 256, 1, "asym"),
                                                     (2, 640, 4104, 10, "asym")])
def test_qdq_warps_match_the_qdq_kernel(M, K, N, n_grid, quantizer, monkeypatch):
    # bf16 W with group 128: the candidate operands are made by the loss GEMM's own QDQ
    # warps while its tensor cores run (the reference launch makes the reference operand
    # and claims candidate tiles while its GEMM runs, the candidate launch the rest);
    # AWQ_QDQ=standalone makes them with qdq_kernel first. Both match the oracle and give
    # the same bits everywhere, tile errors included.
    assert awq.qdq_in_loss_gemm(M, K, N, n_grid) == (awq.loss_gemm_variant(M, K, N, n_grid) == 1)
    spec = custom_spec(M, K, N, group=128, n_grid=n_grid, seed=M + 5 * K + N)
    X, W = generate(spec)
    outs = {}
    for qdq in ("standalone", "warps"):
        if qdq == "standalone":
            monkeypatch.setenv("AWQ_QDQ", "standalone")
        else:
            monkeypatch.delenv("AWQ_QDQ", raising=False)
        if quantizer == "asym":
            P.full_parity(X, W, 128, n_grid)
        outs[qdq] = awq.search(X.cuda(), W.cuda(), 128, n_grid, tile_sq_err=quantizer == "asym", quantizer=quantizer)
    for name in ("scales", "codes", "steps", "zeros", "losses", "best_index") + (("tile_sq_err",) if quantizer == "asym"
                                                                               else ()):
        assert torch.equal(getattr(outs["standalone"], name), getattr(outs["warps"], name)), name


def test_weights_on_the_grid_give_zero_loss():
    # every (group, column) spans all 16 levels with step 1/16 and zero 7: alpha = 0
    # reproduces W exactly (AWQ-P1 §7 reconstruction), so L_0 = 0 and alpha 0 wins
    rng = np.random.default_rng(1)
    K, N, group = 256, 512, 128
    q = rng.integers(0, 16, size=(K, N))
    q[0::group] = 0
    q[1::group] = 15
    W = torch.from_numpy(((q - 7) / 16.0).astype(np.float32)).to(torch.bfloat16)
    X = torch.randn(192, K).to(torch.bfloat16)
    gpu = P.run_gpu(X, W, group, 20)
    assert gpu["losses"][0] == 0.0 and gpu["best"] == 0
    assert np.array_equal(O.unpack_codes(gpu["codes"], N), q)


def test_constant_groups_take_step_one():
    # all-equal groups (AWQ-P1 §7's positive lower bound; step 1 here). With a single
    # candidate alpha = 0 the scales are all 1, so every group of W' stays constant.
    K, N, group = 128, 16, 128
    W = torch.full((K, N), 0.25).to(torch.bfloat16)
    W[:, 8:] = -3.0
    X = torch.randn(8, K).to(torch.bfloat16)
    gpu = P.run_gpu(X, W, group, 1)
    orc = O.search(as_f32_numpy(X), as_f32_numpy(W), group=group, n_grid=1)
    assert np.all(gpu["steps"] == 1.0)
    assert gpu["zeros"][0, :8].tolist() == [0.0] * 8 and gpu["zeros"][0, 8:].tolist() == [3.0] * 8
    P.check_artifact(gpu, as_f32_numpy(W), orc.S, group)


def test_results_are_deterministic():
    spec = custom_spec(256, 512, 768, seed=5)
    X, W = generate(spec)
    a = awq.search(X.cuda(), W.cuda(), tile_sq_err=True)
    b = awq.search(X.cuda(), W.cuda(), tile_sq_err=True)
    for name in ("scales", "codes", "steps", "zeros", "losses", "best_index", "tile_sq_err"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name


def test_host_entry_point_matches_device_entry_point():
    spec = custom_spec(256, 384, 520, seed=9)
    X, W = generate(spec)
    d = awq.search(X.cuda(), W.cuda())
    h = awq.search_host(X.pin_memory(), W.pin_memory())
    for name in ("scales", "codes", "steps", "zeros", "losses", "best_index"):
        assert torch.equal(getattr(d, name).cpu(), getattr(h, name)), name


@pytest.mark.parametrize("dtype,group", [("bf16", 128), ("f32", 64)])
def test_host_batch_matches_one_layer_at_a_time(dtype, group):
    """Five layers through the batched host entry point (inputs of layer i + 1 uploaded
    while layer i runs, two device slots reused) give each layer's own artifact."""
    layers = [generate(custom_spec(256, 384, 520, dtype=dtype, group=group, seed=20 + i)) for i in range(5)]
    outs = awq.search_host_batch([X.pin_memory() for X, _ in layers], [W.pin_memory() for _, W in layers],
                                 group)
    for (X, W), o in zip(layers, outs):
        d = awq.search(X.cuda(), W.cuda(), group)
        for name in ("scales", "codes", "steps", "zeros", "losses", "best_index"):
            assert torch.equal(getattr(d, name).cpu(), getattr(o, name)), name


def test_host_batch_reports_a_bad_layer_and_finishes_the_others():
    layers = [generate(custom_spec(128, 256, 264, seed=40 + i)) for i in range(3)]
    Xs = [X.pin_memory() for X, _ in layers]
    Xs[1][3, 5] = float("nan")
    outs = [awq._alloc_outputs(256, 264, 128, 20, None, pin=True) for _ in range(3)]
    with pytest.raises(awq.AwqError) as e:
        awq.search_host_batch(Xs, [W.pin_memory() for _, W in layers], outs=outs)
    assert e.value.status == 3
    for i in (0, 2):
        d = awq.search(layers[i][0].cuda(), layers[i][1].cuda())
        assert torch.equal(d.codes.cpu(), outs[i][1]) and torch.equal(d.scales.cpu(), outs[i][0])


def test_nonfinite_inputs_are_rejected():
    spec = custom_spec(64, 128, 64, seed=3)
    X, W = generate(spec)
    Xn = X.clone()
    Xn[5, 7] = float("nan")
    with pytest.raises(awq.AwqError) as e:
        awq.search(Xn.cuda(), W.cuda())
    assert e.value.status == 3
    Wn = W.clone()
    Wn[3, 2] = float("inf")
    with pytest.raises(awq.AwqError) as e:
        awq.search(X.cuda(), Wn.cuda())
    assert e.value.status == 3
    # the context stays usable
    awq.search(X.cuda(), W.cuda())


def test_async_searches_back_to_back_match_the_synchronous_call():
    """Four layers enqueued through search_async without waiting (different shapes and
    dtypes on one stream), then waited for: each gives the synchronous call's artifact and
    losses bit for bit, and profiled calls keep their own phase times."""
    specs = [custom_spec(256, 384, 520, seed=50), custom_spec(300, 256, 264, dtype="f32", group=64, seed=51),
             custom_spec(128, 512, 128, seed=52), custom_spec(256, 384, 520, seed=53)]
    layers = [tuple(t.cuda() for t in generate(s)) for s in specs]
    awq.profile_enable(True)
    try:
        pend = [awq.search_async(X, W, s.group, s.n_grid) for s, (X, W) in zip(specs, layers)]
        outs = [p.wait() for p in pend]
        profs = [p.profile() for p in pend]
    finally:
        awq.profile_enable(False)
    for s, (X, W), o, prof in zip(specs, layers, outs, profs):
        d = awq.search(X, W, s.group, s.n_grid)
        for name in ("scales", "codes", "steps", "zeros", "losses", "best_index"):
            assert torch.equal(getattr(d, name), getattr(o, name)), (s.name, name)
        assert set(prof) >= {"statistic", "qdq", "gemm_loss", "pack"}
        assert all(v >= 0.0 for v in prof.values()) and prof["gemm_loss"] > 0.0


def test_unprofiled_async_call_has_no_phase_times():
    spec = custom_spec(128, 256, 264, seed=54)
    X, W = (t.cuda() for t in generate(spec))
    awq.profile_enable(True)
    try:
        awq.search_async(X, W).wait()
    finally:
        awq.profile_enable(False)
    p = awq.search_async(X, W)
    p.wait()
    with pytest.raises(RuntimeError):
        p.profile()


def test_async_search_reports_kernel_errors_on_wait():
    spec = custom_spec(64, 128, 64, seed=3)
    X, W = generate(spec)
    Xn = X.clone()
    Xn[5, 7] = float("nan")
    bad = awq.search_async(Xn.cuda(), W.cuda())
    good = awq.search_async(X.cuda(), W.cuda())
    with pytest.raises(awq.AwqError) as e:
        bad.wait()
    assert e.value.status == 3
    ref = awq.search(X.cuda(), W.cuda())
    assert torch.equal(good.wait().codes, ref.codes)


def test_async_search_needs_a_pinned_status_word():
    import ctypes
    lib = awq.library()
    X = torch.zeros(16, 128, dtype=torch.bfloat16, device="cuda")
    W = torch.zeros(128, 64, dtype=torch.bfloat16, device="cuda")
    outs = awq._alloc_outputs(128, 64, 128, 20, X.device)
    word = (ctypes.c_int32 * 1)()  # pageable host memory
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    st = lib.awq_search_async(p(X), p(W), 0, 16, 128, 64, 128, 20, p(outs[0]), p(outs[1]), p(outs[2]), p(outs[3]),
                              p(outs[4]), p(outs[5]), ctypes.cast(word, ctypes.c_void_p),
                              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 1  # AWQ_ERR_INVALID_ARG


def test_host_pointer_is_rejected_by_the_device_entry_point():
    import ctypes
    lib = awq.library()
    X = torch.zeros(16, 128, dtype=torch.bfloat16)   # host memory
    W = torch.zeros(128, 64, dtype=torch.bfloat16, device="cuda")
    outs = [torch.empty(n, device="cuda", dtype=torch.float32) for n in (128, 128 * 8, 64, 64)]
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    st = lib.awq_search(p(X), p(W), 16, 128, 64, 128, 20, p(outs[0]), p(outs[1]), p(outs[2]), p(outs[3]),
                        ctypes.c_void_p(0), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 1


@pytest.mark.parametrize("qdq", ["warps", "standalone"])
def test_launch_count_and_profile(qdq, monkeypatch):
    if qdq == "standalone":
        monkeypatch.setenv("AWQ_QDQ", "standalone")
    else:
        monkeypatch.delenv("AWQ_QDQ", raising=False)
    spec = custom_spec(256, 256, 512, seed=2)   # bf16, group 128
    X, W = generate(spec)
    awq.profile_enable(True)
    try:
        awq.search(X.cuda(), W.cuda())
        prof = awq.profile_last()
    finally:
        awq.profile_enable(False)
    # statistic + scales + qdq (the reference operand alone when the loss GEMM's QDQ warps
    # make the candidates') + one GEMM launch for the reference output and the candidates
    # (two when the reference has its own launch, always with the QDQ warps) + reduce + pack
    gemm = awq.loss_gemm_launches(256, 256, 512, 20)
    qdq_warps = awq.qdq_in_loss_gemm(256, 256, 512, 20)
    assert qdq_warps == (qdq == "warps" and awq.loss_gemm_variant(256, 256, 512, 20) == 1)
    assert gemm == 2 or not qdq_warps
    assert awq.last_launch_count() == 5 + gemm
    assert set(prof) >= {"statistic", "scales", "qdq", "gemm_reference", "gemm_loss", "loss_reduce", "pack"}
    assert all(v >= 0 for v in prof.values()) and prof["gemm_loss"] > 0


def test_async_search_on_a_side_stream_with_a_non_contiguous_input():
    """An explicit side stream first waits for the current stream, where the inputs and
    their contiguous copies are produced: X is a transposed view whose contiguous copy is
    made on the current stream just before the call. The result equals search()'s bit
    for bit."""
    spec = custom_spec(256, 384, 520, seed=71)
    X, W = (t.cuda() for t in generate(spec))
    ref = awq.search(X, W, spec.group, spec.n_grid)
    Xt = X.t().contiguous()          # (K, M) storage; Xt.t() is X as a non-contiguous view
    side = torch.cuda.Stream()
    torch.cuda._sleep(2_000_000)     # keeps the current stream busy while the call is enqueued
    Xv = Xt.t()
    assert not Xv.is_contiguous()
    out = awq.search_async(Xv, W, spec.group, spec.n_grid, stream=side).wait()
    for name in ("scales", "codes", "steps", "zeros", "losses", "best_index"):
        assert torch.equal(getattr(ref, name), getattr(out, name)), name


def test_the_callers_current_device_is_given_back():
    """A call on a stream of another device runs there and leaves the caller's current
    device as it was."""
    if torch.cuda.device_count() < 2:
        pytest.skip("needs two GPUs")
    spec = custom_spec(128, 256, 264, seed=72)
    X, W = (t.to("cuda:1") for t in generate(spec))
    torch.cuda.set_device(0)
    out = awq.search(X, W, spec.group, spec.n_grid, stream=torch.cuda.Stream(device=1))
    assert torch.cuda.current_device() == 0
    assert out.codes.device == X.device


def test_library_index_is_the_first_minimum_of_tied_losses():
    """An all-zero layer ties every candidate at loss 0: the library keeps the first
    index (AWQ-P1 §3)."""
    K, N = 128, 64
    X = torch.zeros(16, K, dtype=torch.bfloat16, device="cuda")
    W = torch.zeros(K, N, dtype=torch.bfloat16, device="cuda")
    out = awq.search(X, W, 128, 20)
    assert torch.all(out.losses == 0.0)
    assert out.best == 0

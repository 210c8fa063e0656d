"""The C ABI from a plain C program (B200 only).

tests/c/awq_client.c reads a layer from a file, runs it through awq_search_ex,
awq_search_async + awq_search_status and awq_search_host with the CUDA runtime's own
allocations and stream, and writes the results. All three must equal the Python
binding's result bit for bit, and the artifact at the chosen alpha must equal the
oracle's.
"""
import numpy as np
import pytest
import torch

import oracle as O
import post_quantization_column_b200 as awq
from tests import c_client
from tests.parity import check_alpha
from workloads import custom_spec, generate, as_f32_numpy

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,group", [("bf16", 128), ("f32", 64)])
def test_c_client_matches_the_binding_and_the_oracle(dtype, group, tmp_path):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    if not c_client.compiler():
        pytest.skip("no C compiler")
    spec = custom_spec(200, 384, 264, dtype=dtype, group=group, seed=61)
    X, W = generate(spec)
    raw = (lambda t: t.view(torch.int16).numpy().view(np.uint16)) if dtype == "bf16" else (lambda t: t.numpy())
    exe = c_client.build(str(tmp_path))
    c_client.write_input(str(tmp_path / "in.bin"), raw(X), raw(W), group, spec.n_grid, 0 if dtype == "bf16" else 1)
    import subprocess
    run = subprocess.run([exe, str(tmp_path / "in.bin"), str(tmp_path / "out.bin")], capture_output=True, text=True)
    assert run.returncode == 0, run.stderr
    recs = c_client.read_output(str(tmp_path / "out.bin"), spec.K, spec.N, group, spec.n_grid)

    ref = awq.search(X.cuda(), W.cuda(), group, spec.n_grid)
    want = {"scales": ref.scales.cpu().numpy(), "codes": ref.codes.cpu().numpy(),
            "steps": ref.steps.cpu().view(torch.int16).numpy().view(np.uint16),
            "zeros": ref.zeros.cpu().view(torch.int16).numpy().view(np.uint16), "losses": ref.losses.cpu().numpy(),
            "best": ref.best_index.cpu().numpy()}
    for call, rec in zip(("awq_search_ex", "awq_search_async", "awq_search_host"), recs):
        assert rec["status"] == 0, call
        for name, value in want.items():
            assert np.array_equal(rec[name].view(np.uint8), value.view(np.uint8)), (call, name)

    # the index the library returned (out_best) follows the oracle's rule on the losses
    # it returned (AWQ-P1 §3: the first minimum), and the artifact at that alpha is the
    # oracle's
    X32, W32 = as_f32_numpy(X), as_f32_numpy(W)
    best = int(recs[0]["best"][0])
    assert best == int(np.argmin(recs[0]["losses"]))
    r = O.search(X32, W32, group=group, n_grid=spec.n_grid)
    check_alpha(best, r.losses)
    s = O.candidate_scales(O.activation_statistic(X32), spec.n_grid)[best]
    assert np.array_equal(recs[0]["scales"].view(np.uint32), s.view(np.uint32))
    q, step, zero, _ = O.asym_qdq(O.scale_weights(W32, s), group)
    assert np.array_equal(recs[0]["codes"], O.pack_codes(q))
    assert np.array_equal(recs[0]["steps"], O.fp16_rne(step).view(np.uint16))
    assert np.array_equal(recs[0]["zeros"], zero.astype(np.float16).view(np.uint16))

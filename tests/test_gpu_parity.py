"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle on
the same seeded inputs, element by element, max|x-r|/max(1,|r|) <= 5e-3 (fp32
inputs) or 2e-2 (bf16 inputs, fp32 accumulation and state)."""
import pytest
import torch

from tests.parity import assert_parity, run_case

pytestmark = pytest.mark.gpu

BF16, F32 = torch.bfloat16, torch.float32


# ---- the five workload configurations -------------------------------------------------

@pytest.mark.parametrize("seed", [0, 1, 2])
def test_config1_fp32_forward(seed):
    """fp32 forward, B=1 H=1 T=256 d_k=d_v=64, C=64, z~N(0,1)."""
    errs = run_case(1, 1, 256, 64, 64, dtype=F32, chunk=64, seed=seed, bwd=False)
    assert_parity(errs, F32)


@pytest.mark.parametrize("gate", ["vector", "none"])
@pytest.mark.parametrize("variant", ["fused", "materialized"])
def test_config2_bf16_forward(gate, variant):
    """bf16 forward, 340M-layer shape: B=8 H=4 T=2048 d_k=128 d_v=256 C=64 c=16;
    vector gates and the alpha == 1 variant."""
    errs = run_case(8, 4, 2048, 128, 256, dtype=BF16, gate=gate, chunk=64, bwd=False, variant=variant)
    assert_parity(errs, BF16)


def test_config3_bf16_fwd_bwd():
    """bf16 forward + backward, B=8 H=4 T=2048 d_k=128 d_v=256, do~N(0,1)."""
    errs = run_case(8, 4, 2048, 128, 256, dtype=BF16, gate="vector", chunk=64, bwd=True)
    assert_parity(errs, BF16)


@pytest.mark.parametrize("variant", ["fused", "materialized"])
def test_config4_bf16_fwd_bwd(variant):
    """bf16 forward + backward, 1.3B-layer shape: B=2 H=4 T=4096 d_k=256 d_v=512,
    z~N(-1,1)."""
    errs = run_case(2, 4, 4096, 256, 512, dtype=BF16, gate="vector", chunk=64, z_mean=-1.0, bwd=True,
                    variant=variant)
    assert_parity(errs, BF16)


def test_config4_bench_launch_configuration():
    """Config 4 at full size, launched as bench.py times it: one workspace shared by
    gla_fwd and gla_bwd, the forward saving its bf16 chunk states and the backward
    reading them and the forward's prep outputs."""
    errs = run_case(2, 4, 4096, 256, 512, dtype=BF16, gate="vector", chunk=64, z_mean=-1.0, bwd=True,
                    reuse_prep=True, save_states=True)
    assert_parity(errs, BF16)


@pytest.mark.parametrize("T", [1024, 2048, 4096, 8192, 16384])
@pytest.mark.parametrize("gate", ["vector", "scalar", "none"])
def test_config5_sweep(T, gate):
    """B*T = 32768, H=4, d_k=256, d_v=512, bf16 fwd+bwd.  The GPU runs the full
    batch; the oracle checks every head of the first and last batch entry."""
    B = 32768 // T
    sample = [0] if B == 1 else [0, B - 1]
    errs = run_case(B, 4, T, 256, 512, dtype=BF16, gate=gate, chunk=64, bwd=True, sample_b=sample)
    assert_parity(errs, BF16)


# ---- edge cases ------------------------------------------------------------------------

@pytest.mark.parametrize("T", [1, 15, 63, 64, 65, 150, 257])
def test_ragged_lengths_bf16(T):
    errs = run_case(1, 2, T, 128, 128, dtype=BF16, chunk=64, seed=3, with_h0=True, with_dh_final=True)
    assert_parity(errs, BF16)


@pytest.mark.parametrize("chunk", [16, 32, 64, 128])
@pytest.mark.parametrize("gate", ["vector", "scalar", "none"])
def test_fp32_chunks_and_gates(chunk, gate):
    errs = run_case(2, 2, 200, 64, 48, dtype=F32, gate=gate, chunk=chunk, seed=4, with_h0=True,
                    with_dh_final=True)
    assert_parity(errs, F32)


@pytest.mark.parametrize("gate", ["scalar", "none"])
def test_gate_modes_bf16(gate):
    errs = run_case(2, 2, 520, 256, 256, dtype=BF16, gate=gate, chunk=64, seed=5, with_h0=True,
                    with_dh_final=True)
    assert_parity(errs, BF16)


def test_gate_exactly_one_bf16():
    """alpha -> 1: log_alpha == 0 in the vector mode gives ungated attention."""
    errs = run_case(1, 2, 300, 128, 128, dtype=BF16, gate="vector", chunk=64, log_alpha_const=0.0)
    assert_parity(errs, BF16)


def test_strong_gates_bf16():
    """log_alpha = -5 everywhere: whole chunks decay by e^-320, so only the
    sub-chunk rescaling keeps every factor finite."""
    errs = run_case(1, 2, 200, 128, 128, dtype=BF16, gate="vector", chunk=64, log_alpha_const=-5.0,
                    with_h0=True, with_dh_final=True)
    assert_parity(errs, BF16)


def test_strong_gates_fp32():
    errs = run_case(1, 2, 200, 64, 64, dtype=F32, gate="vector", chunk=64, log_alpha_const=-5.0,
                    with_h0=True, with_dh_final=True)
    assert_parity(errs, F32)


@pytest.mark.parametrize("segments", [1, 2, 3, 7])
def test_segment_counts_bf16(segments):
    """The segment-parallel forward gives the same result for any segment count."""
    errs = run_case(2, 2, 1000, 128, 256, dtype=BF16, chunk=64, seed=6, with_h0=True, bwd=False,
                    variant="fused", segments=segments)
    assert_parity(errs, BF16)


def test_h0_and_dh_final_bf16_large_dims():
    errs = run_case(1, 3, 700, 256, 512, dtype=BF16, chunk=64, seed=7, with_h0=True, with_dh_final=True)
    assert_parity(errs, BF16)


@pytest.mark.parametrize("gate", ["vector", "scalar"])
def test_backward_reusing_forward_prep(gate):
    """gla_bwd with GLA_FLAG_REUSE_PREP on the workspace its gla_fwd filled."""
    errs = run_case(2, 2, 777, 256, 512, dtype=BF16, gate=gate, chunk=64, seed=8, with_h0=True,
                    with_dh_final=True, reuse_prep=True)
    assert_parity(errs, BF16)


@pytest.mark.parametrize("variant,segments,reuse_prep", [("fused", 0, True), ("fused", 3, False),
                                                         ("fused", 1, True), ("materialized", 0, True)])
def test_backward_reading_saved_states(variant, segments, reuse_prep):
    """gla_fwd with GLA_FLAG_SAVE_STATES stores the chunk states; gla_bwd with the
    same flag reads them instead of recomputing them."""
    errs = run_case(2, 2, 777, 256, 512, dtype=BF16, gate="vector", chunk=64, seed=9, with_h0=True,
                    with_dh_final=True, variant=variant, segments=segments, reuse_prep=reuse_prep,
                    save_states=True)
    assert_parity(errs, BF16)


def test_saved_states_k128():
    errs = run_case(1, 3, 300, 128, 256, dtype=BF16, gate="scalar", chunk=64, seed=10, with_h0=True,
                    reuse_prep=True, save_states=True)
    assert_parity(errs, BF16)


@pytest.mark.parametrize("chunk,K,V", [(16, 128, 128), (32, 128, 256), (128, 256, 128), (64, 64, 96)])
def test_bf16_shapes_on_the_cuda_core_path(chunk, K, V):
    """bf16 inputs in shapes the tensor-core path does not take (chunk 16, 32 or 128;
    d_k = 64 with d_v = 96) run on the CUDA-core path: fwd+bwd parity at the bf16
    tolerance, ragged T."""
    errs = run_case(1, 2, 300, K, V, dtype=BF16, gate="vector", chunk=chunk, bwd=True, seed=chunk + K)
    assert_parity(errs, BF16)

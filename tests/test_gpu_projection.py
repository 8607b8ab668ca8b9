"""The single-projection workload (X[256 x 512], W[512 x 512], LoRA r 16, alpha 32)
as bench.py --workload single runs it: PactProjection's step, captured into one
CUDA graph with the LoRA weight gradients on a parallel branch, against the oracle's
OracleProjection on the same seeded inputs (NVFP4 copy of X bit-exact; Y, dX, dA
and dB within |gpu - oracle| <= 8e-3 |oracle| + 1e-3 rms(oracle)).  Also: the
activation bytes PyTorch autograd keeps for a plain BF16 LoRA layer, measured with
saved-tensor hooks, against the PACT layer's saved copies."""
import pytest
import torch

import synth
from tests.util import assert_close, assert_nvfp4_equal, to_dev, to_f64

pytestmark = pytest.mark.gpu


def test_single_projection_step_matches_the_oracle(orc):
    import nvfp4_gemm_b200 as P
    from nvfp4_gemm_b200.layer import PactProjection
    from oracle.layer import OracleProjection
    inp = synth.single_inputs()
    M = synth.SINGLE["M"]
    L = PactProjection(to_dev(inp["w"]), to_dev(inp["lora_a"]), to_dev(inp["lora_b"]), M, synth.LORA_R,
                       synth.LORA_ALPHA)
    L.bind(to_dev(inp["x"]), to_dev(inp["dy"]))
    L.step()
    torch.cuda.synchronize()
    s, side = torch.cuda.Stream(), torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        L.step_concurrent(side)
    g.replay()
    torch.cuda.synchronize()
    assert P.pact_get_device_status() == 0, P.pact_last_error()
    ref = OracleProjection(inp["w"], inp["lora_a"], inp["lora_b"], synth.LORA_R, synth.LORA_ALPHA)
    o = ref.step(inp["x"], inp["dy"])
    assert_nvfp4_equal(L.xq, orc.quantize(inp["x"]), orc, "xq")
    wf, wb = orc.weight_cache(inp["w"])
    s_ = synth.LORA_ALPHA / synth.LORA_R
    assert_close(to_f64(L.y), orc.frozen_fwd(orc.quantize(inp["x"]), wf, inp["x"], inp["lora_a"], inp["lora_b"], s_),
                 "Y")
    assert_close(to_f64(L.dx), orc.frozen_dgrad(inp["dy"], wb, inp["lora_a"], inp["lora_b"], s_), "dX")
    assert_close(to_f64(L.grads["a"]), o["dA"], "dA")
    assert_close(to_f64(L.grads["b"]), o["dB"], "dB")


def test_bf16_lora_autograd_saves_more_than_pact():
    import bench
    import oracle
    name, M = "llama-3.2-1b", 256
    c = synth.LAYERS[name]
    measured = bench.bf16_lora_saved_bytes_measured(name, torch.device("cuda"), M)
    model = bench.bf16_lora_saved_bytes(M, c["H"], c["I"], synth.LORA_R)
    pact = oracle.saved_bytes_pact(M, c["H"], c["I"])
    # autograd keeps at least the tensors of the hand count (it may keep more, e.g. silu(gate))
    assert measured >= model > pact
    assert measured <= model + 4 * M * c["I"] * 2, (measured, model)
    torch.cuda.empty_cache()

"""A whole decoder layer (forward + backward) on the GPU against the oracle, stage by
stage.  Each stage is teacher-forced: the oracle stage runs on the GPU's own
upstream tensors, so a legitimate NVFP4 code flip upstream cannot masquerade as an
error downstream.  NVFP4 codes/scales and BF16 values the method rounds exactly
(RMSNorm and SiLU-multiply outputs) must match bit for bit; GEMM and LoRA outputs
must satisfy |gpu - oracle| <= 8e-3 |oracle| + 1e-3 rms(oracle).

The full-size case runs the bench's workload (Llama-3.2-3B layer, 8192 tokens) in
the launch configuration bench.py times (the same op list captured into one CUDA
graph, the LoRA weight gradients on a parallel branch); the frozen GEMM outputs are
checked on sampled rows the oracle computes one by one, everything else in full,
and the graph's results must equal an eager sequential step bit for bit.

With the SiLU-multiply fused into the gate|up GEMM, g|u never reaches memory; the
check recomputes it with the plain GEMM call on the layer's own xq2 and T, which
issues the same tensor-core instructions per tile and so yields the same bits, and
then holds m, mq, gq, uq to the oracle's SiLU-multiply of those bits."""
import numpy as np
import pytest
import torch

import synth
from tests.util import assert_close, assert_nvfp4_equal, to_bits, to_f64

pytestmark = pytest.mark.gpu


def _nv_host(t):
    return t.codes.cpu().numpy(), t.scales.cpu().numpy()


def _bits(t):
    return to_bits(t)


def run_layer(name, M, graphs, two_level=False, fuse_silu=False):
    import nvfp4_gemm_b200 as P
    from nvfp4_gemm_b200.layer import LayerShape, PactLayer
    c = synth.LAYERS[name]
    inp = synth.layer_inputs(name, M=M)
    dev = torch.device("cuda")
    d = lambda b: torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16).to(dev)
    shape = LayerShape(M=M, H=c["H"], I=c["I"], KV=c["KV"])
    L = PactLayer(shape, {k: d(v) for k, v in inp["w"].items()}, {k: d(v) for k, v in inp["lora_a"].items()},
                  {k: d(v) for k, v in inp["lora_b"].items()}, d(inp["gamma1"]), d(inp["gamma2"]),
                  two_level=two_level, fuse_silu=fuse_silu)
    L.bind(d(inp["h"]), d(inp["attn"]), d(inp["d_out"]), d(inp["d_qkv"]))
    ops = L.step_ops()
    if graphs:
        L.step()                       # eager pass first (lazy per-device setup)
        torch.cuda.synchronize()
        # bench.py's timed configuration: the whole step in one CUDA graph, the LoRA
        # weight-gradient leaves on a parallel branch
        s, side = torch.cuda.Stream(), torch.cuda.Stream()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            L.step_concurrent(side)
        for _ in range(2):
            g.replay()
    else:
        L.step()
    torch.cuda.synchronize()
    assert P.pact_get_device_status() == 0, P.pact_last_error()
    return L, inp


def check_layer(L, inp, orc, rows):
    """Teacher-forced stage checks; GEMM outputs on `rows` (None = all rows).  With a
    two-level layer, group k's GEMM outputs are 2^g (frozen + LoRA activations . W),
    its T and U carry s 2^-g and dA is scaled back by 2^g (g = L.gexp[k])."""
    S = L.s
    H, I, KV, r, s = S.H, S.I, S.KV, S.r, S.scale
    f = synth.bf16_bits_to_f64
    sel = slice(None) if rows is None else rows
    cat = lambda names, dct: np.concatenate([dct[n] for n in names], 0)
    wf, wb, ge = {}, {}, {}
    for key, names in (("qkv", ("q", "k", "v")), ("o", ("o",)), ("gu", ("gate", "up")), ("d", ("down",))):
        if L.two_level:
            ge[key], wf[key], wb[key] = orc.weight_cache_two_level(cat(names, inp["w"]))
        else:
            ge[key] = 0
            wf[key], wb[key] = orc.weight_cache(cat(names, inp["w"]))
    assert ge == L.gexp
    p2 = {k: 2.0 ** g for k, g in ge.items()}
    sc = {k: s / p2[k] for k in ge}
    A = {"qkv": f(cat(("q", "k", "v"), inp["lora_a"])), "o": f(inp["lora_a"]["o"]),
         "gu": f(cat(("gate", "up"), inp["lora_a"])), "d": f(inp["lora_a"]["down"])}
    B = {"qkv": f(cat(("q", "k", "v"), inp["lora_b"])), "o": f(inp["lora_b"]["o"]),
         "gu": f(cat(("gate", "up"), inp["lora_b"])), "d": f(inp["lora_b"]["down"])}
    seg = {"qkv": L.seg_qkv, "o": [H], "gu": L.seg_gu, "d": [H]}

    def hilo(t):
        R = t.shape[1] // 2
        return to_f64(t[:, :R]) + to_f64(t[:, R:])

    def nv_equal(dev_t, ref_t, what):
        assert_nvfp4_equal(dev_t, ref_t, orc, what)

    def gemm_rows(aq_ref, w):
        a = aq_ref if rows is None else aq_ref.rows_slice(rows)
        return orc.nvfp4_gemm(a, w)

    def lora_rows(act_dev, key, fwd):
        act = act_dev[sel]
        out = np.zeros((act.shape[0], seg[key][-1] if fwd else A[key].shape[1]))
        lo = 0
        for i, hi in enumerate(seg[key] if fwd else [A[key].shape[0] // r]):
            if fwd:
                out[:, lo:hi] = orc.gemm_nt(act[:, i * r:(i + 1) * r], B[key][lo:hi])
                lo = hi
        if not fwd:
            out = orc.gemm_nt(act, A[key].T)
        return out

    def lora_grads_tf(dy_bits, xt, u_dev, key, gA, gB, what):
        dy = f(dy_bits)
        assert_close(to_f64(gA), p2[key] * orc.gemm_nt(u_dev.T, xt.T), f"dA {what}")
        db = np.zeros_like(B[key])
        lo = 0
        for i, hi in enumerate(seg[key]):
            db[lo:hi] = s * orc.gemm_nt(dy[:, lo:hi].T, orc.gemm_nt(xt, A[key][i * r:(i + 1) * r]).T)
            lo = hi
        assert_close(to_f64(gB), db, f"dB {what}")

    def u_ref(dy_bits, key):
        dy = f(dy_bits)
        out = np.zeros((dy.shape[0], len(seg[key]) * r))
        lo = 0
        for i, hi in enumerate(seg[key]):
            out[:, i * r:(i + 1) * r] = sc[key] * orc.gemm_nt(dy[:, lo:hi], B[key][lo:hi].T)
            lo = hi
        return out

    h, attn, d_out, d_qkv = inp["h"], inp["attn"], inp["d_out"], inp["d_qkv"]
    # ---- forward
    y1, xq1, rstd1 = orc.rmsnorm_quant(h, inp["gamma1"], S.eps)
    assert np.array_equal(_bits(L.x1), y1), "x1"
    nv_equal(L.xq1, xq1, "xq1")
    np.testing.assert_allclose(L.rstd1.cpu().numpy(), rstd1, rtol=1e-7)
    t_qkv = hilo(L.t_qkv)
    assert_close(t_qkv, sc["qkv"] * orc.gemm_nt(f(y1), A["qkv"]), "T qkv")
    assert_close(to_f64(L.qkv)[sel], p2["qkv"] * (gemm_rows(xq1, wf["qkv"]) + lora_rows(t_qkv, "qkv", True)), "qkv")
    aq = orc.quantize(attn)
    nv_equal(L.aq, aq, "q(attn)")
    t_o = hilo(L.t_o)
    assert_close(t_o, sc["o"] * orc.gemm_nt(f(attn), A["o"]), "T o")
    assert_close(to_f64(L.h2)[sel], f(h)[sel] + p2["o"] * (gemm_rows(aq, wf["o"]) + lora_rows(t_o, "o", True)),
                 "h2")
    h2 = _bits(L.h2)
    y2, xq2, rstd2 = orc.rmsnorm_quant(h2, inp["gamma2"], S.eps)
    assert np.array_equal(_bits(L.x2), y2), "x2"
    nv_equal(L.xq2, xq2, "xq2")
    t_gu = hilo(L.t_gu)
    assert_close(t_gu, sc["gu"] * orc.gemm_nt(f(y2), A["gu"]), "T gu")
    if L.gu is None:
        import nvfp4_gemm_b200 as P
        gu_dev = P.pact_frozen_gemm_fwd(L.xq2, L.c_gu, L.l_gu_f)
        torch.cuda.synchronize()
    else:
        gu_dev = L.gu
    assert_close(to_f64(gu_dev)[sel], p2["gu"] * (gemm_rows(xq2, wf["gu"]) + lora_rows(t_gu, "gu", True)),
                 "gate|up")
    gu = _bits(gu_dev)
    m, mq, gq, uq = orc.silu_mul_quant(gu[:, :I], gu[:, I:])
    if L.m is not None:   # m itself is kept only by the fused SiLU GEMM; the default path checks mq and T down
        assert np.array_equal(_bits(L.m), m), "m"
    nv_equal(L.mq, mq, "mq")
    nv_equal(L.gq, gq, "gq")
    nv_equal(L.uq, uq, "uq")
    t_d = hilo(L.t_d)
    assert_close(t_d, sc["d"] * orc.gemm_nt(f(m), A["d"]), "T down")
    assert_close(to_f64(L.out)[sel], f(h2)[sel] + p2["d"] * (gemm_rows(mq, wf["d"]) + lora_rows(t_d, "d", True)),
                 "out")
    # ---- backward: down
    u_d = hilo(L.u_d)
    assert_close(u_d, u_ref(d_out, "d"), "U down")
    doq = orc.quantize(d_out)
    nv_equal(L.doq, doq, "q(d_out)")
    assert_close(to_f64(L.dm)[sel], p2["d"] * (gemm_rows(doq, wb["d"]) + lora_rows(u_d, "d", False)), "dm")
    dm = _bits(L.dm)
    dg, du = orc.silu_mul_bwd(f(dm), gq, uq)
    dgu_dev = to_f64(L.dgu)
    assert_close(dgu_dev[:, :I], dg, "dg")
    assert_close(dgu_dev[:, I:], du, "du")
    dgu = _bits(L.dgu)
    dguq = orc.quantize(dgu)
    nv_equal(L.dguq, dguq, "q(dg|du)")
    m_re = orc.silu_mul_recompute(gq, uq)
    assert np.array_equal(_bits(L.m_re), m_re), "m~"
    lora_grads_tf(d_out, f(m_re), u_d, "d", L.grads["a_d"], L.grads["b_d"], "down")
    # gate|up
    u_gu = hilo(L.u_gu)
    assert_close(u_gu, u_ref(dgu, "gu"), "U gate|up")
    assert_close(to_f64(L.dx2)[sel], p2["gu"] * (gemm_rows(dguq, wb["gu"]) + lora_rows(u_gu, "gu", False)), "dx2")
    lora_grads_tf(dgu, xq2.dequantize(), u_gu, "gu", L.grads["a_gu"], L.grads["b_gu"], "gate|up")
    dx2 = _bits(L.dx2)
    dh2_ref = orc.rmsnorm_bwd(f(dx2), xq2, L.rstd2.cpu().numpy().astype(np.float64), inp["gamma2"]) + f(d_out)
    assert_close(to_f64(L.dh2), dh2_ref, "dh2")
    dh2 = _bits(L.dh2)
    dh2q = orc.quantize(dh2)
    nv_equal(L.dh2q, dh2q, "q(dh2)")
    # o
    u_o = hilo(L.u_o)
    assert_close(u_o, u_ref(dh2, "o"), "U o")
    assert_close(to_f64(L.dattn)[sel], p2["o"] * (gemm_rows(dh2q, wb["o"]) + lora_rows(u_o, "o", False)), "d attn")
    lora_grads_tf(dh2, f(attn), u_o, "o", L.grads["a_o"], L.grads["b_o"], "o")
    # q|k|v
    u_qkv = hilo(L.u_qkv)
    assert_close(u_qkv, u_ref(d_qkv, "qkv"), "U qkv")
    dqkvq = orc.quantize(d_qkv)
    nv_equal(L.dqkvq, dqkvq, "q(d_qkv)")
    assert_close(to_f64(L.dx1)[sel], p2["qkv"] * (gemm_rows(dqkvq, wb["qkv"]) + lora_rows(u_qkv, "qkv", False)),
                 "dx1")
    lora_grads_tf(d_qkv, xq1.dequantize(), u_qkv, "qkv", L.grads["a_qkv"], L.grads["b_qkv"], "qkv")
    dh_ref = orc.rmsnorm_bwd(f(_bits(L.dx1)), xq1, L.rstd1.cpu().numpy().astype(np.float64),
                             inp["gamma1"]) + f(dh2)
    assert_close(to_f64(L.dh), dh_ref, "dh")


SMALL = {"H": 512, "I": 1024, "KV": 256, "batch": 1, "seq": 300, "outliers": True}


@pytest.fixture
def small_layer(monkeypatch):
    monkeypatch.setitem(synth.LAYERS, "tiny", SMALL)
    return "tiny"


@pytest.mark.parametrize("graphs,fuse", [(False, False), (False, True), (True, True)])
def test_layer_small_all_rows(orc, small_layer, graphs, fuse):
    L, inp = run_layer(small_layer, 300, graphs, fuse_silu=fuse)
    assert L.fuse_silu == fuse
    check_layer(L, inp, orc, rows=None)
    assert L.saved_bytes() == orc.saved_bytes_pact(300, L.s.H, L.s.I)


def test_layer_small_two_level(orc, small_layer):
    """The two-level weight layouts through the whole layer (weights with 1% x20
    outliers), in the bench's launch configuration, all rows."""
    L, inp = run_layer(small_layer, 300, graphs=True, two_level=True)
    assert all(g < 0 for g in L.gexp.values())
    check_layer(L, inp, orc, rows=None)


@pytest.mark.parametrize("name,fuse", [("qwen2.5-1.5b", True), ("llama-3.2-1b", False)])
def test_layer_full_size(orc, name, fuse):
    """The other two layer workloads (Qwen2.5-1.5B, I = 8960 = 35 x 256, with the
    SiLU-multiply in the gate|up GEMM's epilogue, and Llama-3.2-1B, each at 2048
    tokens) in the bench's launch configuration."""
    L, inp = run_layer(name, synth.tokens(name), graphs=True, fuse_silu=fuse)
    assert L.saved_bytes() == orc.saved_bytes_pact(L.s.M, L.s.H, L.s.I)
    rows = np.sort(np.random.default_rng(12).choice(L.s.M, size=32, replace=False))
    rows[-1] = L.s.M - 1
    check_layer(L, inp, orc, rows=rows)


def test_layer_bench_workload_full_size(orc):
    """The bench workload itself (Llama-3.2-3B at 8192 tokens, 1% x20 weight
    outliers), in the bench's launch configuration."""
    L, inp = run_layer("llama-3.2-3b", synth.tokens("llama-3.2-3b"), graphs=True, fuse_silu=False)
    assert not L.fuse_silu and L.saved_bytes() == orc.saved_bytes_pact(L.s.M, L.s.H, L.s.I)
    # the concurrent graph step and an eager sequential step agree bit for bit
    snap = {k: v.clone() for k, v in L.grads.items()}
    outs = {"out": L.out.clone(), "dh": L.dh.clone(), "dattn": L.dattn.clone()}
    L.step()
    torch.cuda.synchronize()
    for k, v in snap.items():
        assert torch.equal(v, L.grads[k]), f"LoRA gradient {k}: concurrent graph step != eager step"
    for k, v in outs.items():
        assert torch.equal(v, getattr(L, k)), f"{k}: concurrent graph step != eager step"
    rows = np.sort(np.random.default_rng(11).choice(L.s.M, size=48, replace=False))
    rows[-1] = L.s.M - 1
    check_layer(L, inp, orc, rows=rows)

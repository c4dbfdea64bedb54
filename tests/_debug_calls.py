"""A representative set of the library's calls on small seeded inputs, used
by the debug-build GPU test to run the same work through the release and the
checked library (no method arithmetic here: inputs and the calls only)."""
import torch

import workloads


def run_all(w8, dev):
    """{name: CPU tensor} of every call's output, in a fixed order."""
    out = {}
    x = lambda M, K, s: workloads.with_outlier_channels((M, K), 1.0, seed=s).to(dev)
    w = lambda N, K, s: workloads.normal((N, K), 0.02, seed=s).to(dev)
    bias = lambda N: workloads.normal((N,), 0.01, seed=N).to(dev)
    # the forward's kernels: few-token (1, 2 rows), transposed (64), split-K
    # (7 x 1000 x 4096), single-SM tiles (200), CTA pairs (600), both formats
    for qt in ("int8", "e4m3"):
        for gran in ("tensor", "axis"):
            wq, sw = w8.quantize_weight(w(1000, 640, 11), qt, gran)
            out["wq_%s_%s" % (qt, gran)] = wq.view(torch.uint8).cpu()
            for M in (1, 2, 64, 200, 600):
                out["fwd_%s_%s_%d" % (qt, gran, M)] = w8.linear_fwd(x(M, 640, M), wq, sw, bias=bias(1000)).cpu()
        wq, sw = w8.quantize_weight(w(1000, 4096, 12), qt, "tensor")
        out["fwd_split_%s" % qt] = w8.linear_fwd(x(7, 4096, 13), wq, sw).cpu()
        wq, sw = w8.quantize_weight(w(528, 512, 14), qt, "tensor")
        for M in (64, 600):
            out["dgrad_%s_%d" % (qt, M)] = w8.linear_dgrad(workloads.normal((M, 528), 1e-3, M).to(dev), wq, sw).cpu()
    # the chain's activation and row absmax
    wq, sw = w8.quantize_weight(w(1024, 512, 15), "int8", "tensor")
    amax = torch.zeros((600,), dtype=torch.int32, device=dev)
    out["fwd_gelu"] = w8.linear_fwd_ex(x(600, 512, 16), wq, sw, act="gelu", y_amax=amax).cpu()
    out["fwd_gelu_amax"] = amax.cpu()
    # row quantizer on long rows (the one-block-per-row kernel)
    q, s = w8.quantize_rows(x(2, 110016, 17), "int8")
    out["rows_q"], out["rows_s"] = q.view(torch.uint8).cpu(), s.cpu()
    # Q8_0: quantize, dequantize (fp32, bf16), requant (hold, team and warp kernels)
    v = workloads.q8_0_standalone(100003, seed=18).to(dev)
    blk = w8.q8_0_quantize(v)
    out["q8_blocks"] = blk.cpu()
    out["q8_deq"] = w8.q8_0_dequantize(blk, 100003).cpu()
    out["q8_deq_bf16"] = w8.q8_0_dequantize_bf16(blk, 100003).cpu()
    for N, K in ((50, 3072), (12, 4128), (4, 32768)):
        b = w8.q8_0_quantize(workloads.normal((N, K), 0.02, seed=N).float().reshape(-1).to(dev))
        for qt in ("int8", "e4m3"):
            q, s = w8.q8_0_to_axis(b, N, K, qt)
            out["rq_%s_%d_%d" % (qt, N, K)] = q.view(torch.uint8).cpu()
            out["rq_s_%s_%d_%d" % (qt, N, K)] = s.cpu()
    # weight-only types and the bf16 Linear, forward and input gradient
    wq8, sw8 = w8.quantize_weight(w(520, 512, 19), "e4m3", "tensor")
    bq = w8.q8_0_quantize(workloads.normal((520, 512), 0.02, seed=20).float().reshape(-1).to(dev))
    for M in (64, 600):
        out["wo_f8_%d" % M] = w8.float8_linear_fwd(x(M, 512, 21), wq8, sw8).cpu()
        out["wo_gguf_%d" % M] = w8.gguf_linear_fwd(x(M, 512, 22), bq, 520).cpu()
        dy = workloads.normal((M, 520), 1e-3, seed=23).to(dev)
        out["wo_f8_dgrad_%d" % M] = w8.float8_linear_dgrad(dy, wq8, sw8).cpu()
        out["wo_gguf_dgrad_%d" % M] = w8.gguf_linear_dgrad(dy, bq, 512).cpu()
    # SVDQuant, single-SM and CTA-pair forms, both residual formats
    for qt in ("int8", "e4m3"):
        prep = w8.svdq_prepare(workloads.rank_spike_weight(520, 512, 8, 0.5, 0.02, 24).to(dev), 16, qt)
        for M in (200, 600):
            out["svdq_%s_%d" % (qt, M)] = w8.svdq_linear_fwd(x(M, 512, 25), prep["rq"], prep["r_scale"], prep["l1"],
                                                             prep["l2"], bias=bias(520)).cpu()
    # rows longer than the one-pass input kernel holds: row quantizer + T product
    prep = w8.svdq_prepare(workloads.rank_spike_weight(136, 3088, 8, 0.5, 0.02, 26).to(dev), 8, "int8")
    out["svdq_long_rows"] = w8.svdq_linear_fwd(x(45, 3088, 27), prep["rq"], prep["r_scale"], prep["l1"],
                                               prep["l2"]).cpu()
    torch.cuda.synchronize()
    return out

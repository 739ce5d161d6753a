"""Rank bodies of the expert-parallel tests (not collected by pytest on its own).

`cpu_rank` runs one gloo rank on CPU with the layer's steps computed by the oracle; `gpu_main`
runs one NCCL rank (world size 1) with the library's kernels.  Both compare the expert-parallel
forward with the single-batch layer on the union of the ranks' tokens.
"""
import math
import os
import sys

import numpy as np
import torch
import torch.distributed as dist

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from expert_ffn_layer_router_b200 import inputs  # noqa: E402


def _np(t):
    """numpy view of a CPU tensor; bfloat16 as its raw bits (uint16), as the oracle takes it."""
    return t.view(torch.int16).numpy().view(np.uint16) if t.dtype == torch.bfloat16 \
        else t.numpy()


def _t(a):
    """CPU tensor of a numpy array; uint16 bit patterns become bfloat16 values."""
    a = np.ascontiguousarray(a)
    return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) if a.dtype == np.uint16 \
        else torch.from_numpy(a)


class OracleSteps:
    """The layer's steps computed by the oracle on CPU tensors (expert rows travel as float64),
    for checking the expert-parallel exchange on gloo ranks."""

    def __init__(self, T_local, E_local, k, flags):
        self.T_local, self.E_local, self.k, self.flags = T_local, E_local, k, flags

    def route(self, x, Wr, br):
        L = oracle.logits(_np(x), Wr.numpy(), None if br is None else br.numpy())
        r = oracle.route(L, self.k, self.T_local, self.flags & oracle.RENORMALIZE)
        return torch.from_numpy(r["ids"]), torch.from_numpy(r["w"])

    def select(self, e_v, w_v, K):
        n = e_v.shape[0]
        ids = e_v.numpy().reshape(n, 1)
        ro = oracle.select(ids, w_v.numpy().reshape(n, 1), self.E_local, K,
                           self.flags & oracle.ARRIVAL_ORDER)
        offsets, rowtok = oracle.dispatch(ids, ro["slot"], self.E_local)
        return torch.from_numpy(ro["slot"].reshape(n)), torch.from_numpy(offsets), \
            torch.from_numpy(rowtok)

    def expert_ffn(self, x_rows, offsets, rowtok, W1, b1, W2, b2):
        off = offsets.numpy()
        row_exp = np.repeat(np.arange(self.E_local, dtype=np.int32), np.diff(off))
        if row_exp.size == 0:
            return torch.zeros((0, W2.shape[1]), dtype=torch.float64)
        Y = oracle.expert_rows(_np(x_rows), _np(W1), b1.numpy(), _np(W2), b2.numpy(),
                               rowtok.numpy(), row_exp, flags=self.flags & oracle.GATED)
        return torch.from_numpy(Y)

    def combine(self, x, Y_back, w, slot_back):
        # The oracle's order: s = sum over kept j (ascending) of w * y in double, then x + s,
        # rounded once; a token with no kept pair is x unchanged.
        xv = _np(x)
        x64 = inputs.bf16_bits_to_f32(xv).astype(np.float64) if xv.dtype == np.uint16 \
            else xv.astype(np.float64)
        Y = Y_back.numpy()
        wv, sl = w.numpy(), slot_back.numpy()
        T, d = x64.shape
        out64 = np.empty((T, d), np.float64)
        outx = np.empty_like(xv)
        for t in range(T):
            s = np.zeros(d, np.float64)
            any_kept = False
            for j in range(self.k):
                if sl[t, j] >= 0:
                    s += np.float64(wv[t, j]) * Y[sl[t, j]]
                    any_kept = True
            out64[t] = x64[t] + s
            if not any_kept:
                outx[t] = xv[t]
            elif xv.dtype == np.uint16:
                outx[t] = np.array([oracle.bf16_from_double(v) for v in out64[t]], np.uint16)
            else:
                outx[t] = out64[t].astype(np.float32)
        return (torch.from_numpy(out64), _t(outx))


def layer_global(spec, seed):
    return inputs.make_layer(spec, seed=seed)


def cpu_rank(rank, world, port, args, out):
    """One gloo rank: the expert-parallel forward with oracle steps, checked against the
    single-batch oracle forward.  out[rank] = list of failures (empty when equal)."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from expert_ffn_layer_router_b200 import build as lib_build
    lib_build.build()
    from expert_ffn_layer_router_b200.ep import ExpertParallelLayer
    T_l, d, F, E, k, C, dtype, flags, seed = args
    spec = inputs.LayerSpec("ep", T_l * world, d, F, E, k, C, dtype, router="normal",
                            router_bias=0.5, bias_std=0.05)
    L = layer_global(spec, seed)
    ref = oracle.forward(L["x"], L["Wr"], L["br"], L["W1"], L["b1"], L["W2"], L["b2"], k, C,
                         flags=flags)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    fails = []
    try:
        El = E // world
        sl = slice(rank * T_l, (rank + 1) * T_l)
        es = slice(rank * El, (rank + 1) * El)
        ep = ExpertParallelLayer(dist.group.WORLD, T_l, d, F, E, k, C, dtype, "cpu", flags,
                                 steps=OracleSteps(T_l, El, k, flags))
        if ep.K != ref["K"]:
            fails.append("capacity %d != %d" % (ep.K, ref["K"]))
        (out64, outx), r = ep.forward(_t(L["x"][sl]), torch.from_numpy(L["Wr"]),
                                      torch.from_numpy(L["br"]), _t(L["W1"][es]),
                                      torch.from_numpy(L["b1"][es]), _t(L["W2"][es]),
                                      torch.from_numpy(L["b2"][es]))
        rr = ref["route"]
        for key in ("ids", "slot", "drop"):
            if not np.array_equal(r[key].numpy(), rr[key][sl]):
                fails.append("routing differs: " + key)
        if not np.array_equal(r["w"].numpy().view(np.uint32), rr["w"][sl].view(np.uint32)):
            fails.append("weights differ")
        if not np.array_equal(out64.numpy(), ref["out_f64"][sl]):
            fails.append("float64 outputs differ (max %g)" %
                         np.abs(out64.numpy() - ref["out_f64"][sl]).max())
        if not np.array_equal(_np(outx), ref["out"][sl]):
            fails.append("rounded outputs differ")
        dist.barrier()
    finally:
        dist.destroy_process_group()
    out[rank] = fails


def gpu_main():
    """World size 1 on one GPU (NCCL): the expert-parallel path with every expert local must give
    moe_forward's results bit for bit.  Prints OK or the differences; exit code 0 when equal."""
    import expert_ffn_layer_router_b200.moe as moe
    from expert_ffn_layer_router_b200.ep import ExpertParallelLayer
    T, d, F, E, k, C, dtype, flags = (int(sys.argv[2]), int(sys.argv[3]), int(sys.argv[4]),
                                      int(sys.argv[5]), int(sys.argv[6]), float(sys.argv[7]),
                                      sys.argv[8], int(sys.argv[9]))
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=dev)
    spec = inputs.LayerSpec("ep", T, d, F, E, k, C, dtype, router="normal", router_bias=0.5,
                            bias_std=0.05)
    L = inputs.make_layer(spec, seed=T + E)

    def td(a):
        return _t(a).to(dev)

    args = [td(L[n]) for n in ("x", "Wr", "br", "W1", "b1", "W2", "b2")]
    layer = moe.MoELayer(T, d, F, E, k, C, dtype, flags=flags)
    out_ref, rt = layer.forward(*args, want_routing=True)
    ep = ExpertParallelLayer(dist.group.WORLD, T, d, F, E, k, C, dtype, dev, flags)
    out, r = ep.forward(*args)
    torch.cuda.synchronize()
    bad = []
    for key in ("ids", "slot", "drop"):
        if not torch.equal(r[key], rt[key + "_out"]):
            bad.append(key)
    if not torch.equal(r["w"].view(torch.int32), rt["w_out"].view(torch.int32)):
        bad.append("w")
    if not torch.equal(out.view(torch.int16) if out.dtype == torch.bfloat16 else out,
                       out_ref.view(torch.int16) if out_ref.dtype == torch.bfloat16 else out_ref):
        bad.append("out")
    st = [moe.moe_get_device_status(w) for w in (ep.steps.sel_ws, ep.steps.ffn_ws,
                                                 ep.steps.comb_ws, layer.ws)]
    if any(st):
        bad.append("device status %s" % st)
    dist.destroy_process_group()
    print("OK" if not bad else "DIFF " + " ".join(bad))
    sys.exit(0 if not bad else 1)


if __name__ == "__main__" and len(sys.argv) > 1 and sys.argv[1] == "gpu":
    gpu_main()

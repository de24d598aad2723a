"""Run by tests/test_gpu_debug_build.py in a child process with
ATTN_DEBUG=1 (the binding then loads libb200attn_debug.so): the small and
ragged parity shapes through every attention mode and kernel and the
projection GEMMs, each followed by a status check.  Prints one JSON line per
case: its status and its error against the FP64 oracle."""
import json
import math
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import long_context_bidirectional_b200 as b2a  # noqa: E402
import workloads as W  # noqa: E402
from oracle import attention as OA  # noqa: E402
from oracle import chunked as OC  # noqa: E402
from oracle import stack as OS  # noqa: E402


def status():
    try:
        b2a.check_status()
        return "ok"
    except b2a.B2AError as e:
        return f"{e.status}: {e}"


def err(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.max(np.abs(got - ref))), float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))


def emit(**kw):
    print(json.dumps(kw), flush=True)


def main():
    assert b2a.lib.b2a_debug_build() == 1, "not the debug build"
    torch.cuda.set_device(0)
    kernels = {64: [b2a.ATTN_KERNEL_SINGLE], 128: [b2a.ATTN_KERNEL_SINGLE, b2a.ATTN_KERNEL_PAIR]}
    for S in (1, 3, 127, 129, 1000):
        for d in (64, 128):
            H = 2
            q, k, v = W.qkv(S, H, d, seed=S + d, q_sigma=2.0)
            scale = 1 / math.sqrt(d)
            ref, ref_lse = OA.attention(q, k, v, scale)
            qd, kd, vd = (torch.from_numpy(x).cuda() for x in (q, k, v))
            for kern in kernels[d]:
                b2a.set_attn_kernel(kern)
                try:
                    out, lse = b2a.attn_fwd(qd, kd, vd, scale=scale)
                    st = status()
                    ma, rf = err(out.cpu().numpy(), ref)
                    dl = float(np.max(np.abs(lse.cpu().numpy() - ref_lse)))
                    emit(case=f"attn_fwd S={S} d={d} kernel={kern}", status=st, max_abs=ma, rel_fro=rf, dlse=dl)
                    P = min(3, S)
                    o_p, l_p = b2a.attn_fwd_partials(qd, kd, vd, P, scale=scale)
                    st = status()
                    ro, rl = OC.partials(q, k, v, scale, P)
                    ma, rf = err(o_p.cpu().numpy(), ro)
                    dl = float(np.max(np.abs(l_p.cpu().numpy() - rl)))
                    emit(case=f"attn_fwd_partials S={S} d={d} P={P} kernel={kern}", status=st, max_abs=ma,
                         rel_fro=rf, dlse=dl)
                    out_r, lse_r = b2a.attn_ring(qd, kd, vd, min(2, S), scale=scale)
                    st = status()
                    ma, rf = err(out_r.cpu().numpy(), ref)
                    dl = float(np.max(np.abs(lse_r.cpu().numpy() - ref_lse)))
                    emit(case=f"ring S={S} d={d} kernel={kern}", status=st, max_abs=ma, rel_fro=rf, dlse=dl)
                finally:
                    b2a.set_attn_kernel(b2a.ATTN_KERNEL_AUTO)
    # projection GEMMs on ragged shapes (fused QKV, output with residual, q/k RMSNorm)
    for (M, N, K) in ((1, 384, 64), (129, 768, 136), (1000, 1536, 512)):
        a, w = W.gemm_operands(M, N, K, seed=M)
        y = b2a.qkv_proj(torch.from_numpy(a).cuda(), torch.from_numpy(w).cuda())
        st = status()
        ma, rf = err(y.cpu().numpy(), OS.linear(a, w))
        emit(case=f"qkv_proj {M}x{N}x{K}", status=st, max_abs=ma, rel_fro=rf, dlse=0.0)
        r = torch.from_numpy(a[:, :1].repeat(N, axis=1).copy()).cuda()
        y2 = b2a.out_proj(torch.from_numpy(a).cuda(), torch.from_numpy(w).cuda(), residual=r)
        st = status()
        ma, rf = err(y2.cpu().numpy(), OS.linear(a, w) + a[:, :1].astype(np.float64))
        emit(case=f"out_proj {M}x{N}x{K}", status=st, max_abs=ma, rel_fro=rf, dlse=0.0)
    H, d = 2, 64
    xq, wq = W.gemm_operands(257, 3 * H * d, 128, seed=9)
    g = np.ones(d, dtype=np.float16)
    gd = torch.from_numpy(g).cuda()
    yq = b2a.qkv_proj_qknorm(torch.from_numpy(xq).cuda(), torch.from_numpy(wq).cuda(), gd, gd, H, d, 1e-6)
    st = status()
    ma, rf = err(yq.cpu().numpy(), OS.qkv_qknorm(xq, wq, g, g, H, d, 1e-6))
    emit(case="qkv_proj_qknorm 257 rows", status=st, max_abs=ma, rel_fro=rf, dlse=0.0)


if __name__ == "__main__":
    main()

"""Run one operation of the library on its seeded synthetic workload, for
profilers (ncu) and quick timing: nothing is checked against the oracle here,
only the device status word.

    python -m moe_gemm_token_b200.drive moe   [--calls N]
    python -m moe_gemm_token_b200.drive gemm  M N K [--calls N]
    python -m moe_gemm_token_b200.drive fused M N K [--calls N]
    python -m moe_gemm_token_b200.drive decode M [--calls N]
    python -m moe_gemm_token_b200.drive w16 M N K [--calls N]
    python -m moe_gemm_token_b200.drive w16w M N K [--calls N]
    python -m moe_gemm_token_b200.drive quant M K [--calls N]
    python -m moe_gemm_token_b200.drive moe4  [--calls N]
    python -m moe_gemm_token_b200.drive gemm4 M N K [--calls N]
    python -m moe_gemm_token_b200.drive shared [--calls N]
    python -m moe_gemm_token_b200.drive bf16 M N K [--calls N]

Each call is enqueued on the current stream; the script synchronises once at
the end and exits non-zero if the device status word reports an error.
"""
import argparse
import sys

import torch

from moe_gemm_token_b200 import metis


def _codes(n, k, g):
    c = torch.randint(0, 256, (n, k), dtype=torch.uint8, device="cuda", generator=g)
    c[(c & 0x7F) == 0x7F] = 0x38  # no NaN codes
    return c


def _sf(n, g):
    """E4M3 block scales 2^-3 .. 2^2 (no NaN code), in any layout."""
    return torch.randint(0x20, 0x48, (n,), dtype=torch.uint8, device="cuda", generator=g)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("op", choices=["moe", "gemm", "fused", "decode", "w16", "w16w", "quant", "moe4", "gemm4", "shared",
                                   "bf16"])
    ap.add_argument("dims", nargs="*", type=int)
    ap.add_argument("--calls", type=int, default=3)
    a = ap.parse_args(argv)
    metis.load()
    g = torch.Generator(device="cuda")
    g.manual_seed(7)
    dev = "cuda"
    if a.op in ("moe", "shared"):
        T, H, I, E, k = 4096, 2048, 1024, 64, 8
        x = torch.randn(T, H, device=dev, generator=g).to(torch.bfloat16)
        logits = torch.randn(T, E, device=dev, generator=g)
        logits[:, :4] += 0.93  # four hot experts, about 3x the mean load
        top = torch.topk(logits, k, dim=1)
        ids = top.indices.to(torch.int32).contiguous()
        w = torch.softmax(top.values, dim=1).float().contiguous()
        wu = _codes(E * I, H, g).view(E, I, H)
        su = torch.rand(E, I, device=dev, generator=g) * 1e-3
        wd = _codes(E * H, I, g).view(E, H, I)
        sd = torch.rand(E, H, device=dev, generator=g) * 1e-3
        y = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
        ws = torch.empty(metis.metis_workspace_size(metis.METIS_OP_MOE, T, I, H, k, E),
                         dtype=torch.uint8, device=dev)
        call = lambda: metis.metis_moe_fp8_grouped_gemm(x, ids, w, wu, su, wd, sd, y, ws)
        if a.op == "shared":
            # routed layer with y = NULL, then the BF16 shared expert (latent
            # 1024) with the routed combine fused into its down-projection
            wsu = (torch.randn(1024, H, device=dev, generator=g) * 0.03).to(torch.bfloat16)
            wsd = (torch.randn(H, 1024, device=dev, generator=g) * 0.03).to(torch.bfloat16)
            wss = torch.empty(metis.metis_workspace_size(metis.METIS_OP_SHARED, T, 1024, H, k, 0),
                              dtype=torch.uint8, device=dev)
            o_off = metis.metis_moe_workspace_offset("O", T, k, E, H, I)
            r_off = metis.metis_moe_workspace_offset("SLOT_TO_ROW", T, k, E, H, I)
            o_reg = ws[o_off:].view(torch.bfloat16)
            s2r = ws[r_off:r_off + 4 * T * k].view(torch.int32)

            def call():
                metis.metis_moe_fp8_grouped_gemm(x, ids, w, wu, su, wd, sd, None, ws)
                metis.metis_moe_shared_fused_combine(x, wsu, wsd, o_reg, s2r, w, y, wss)
    elif a.op == "moe4":
        T, H, I, E, k = 4096, 2048, 1024, 64, 8
        x = torch.randn(T, H, device=dev, generator=g).to(torch.bfloat16)
        logits = torch.randn(T, E, device=dev, generator=g)
        logits[:, :4] += 0.93
        top = torch.topk(logits, k, dim=1)
        ids = top.indices.to(torch.int32).contiguous()
        w = torch.softmax(top.values, dim=1).float().contiguous()
        wu = torch.randint(0, 256, (E, I, H // 2), dtype=torch.uint8, device=dev, generator=g)
        wd = torch.randint(0, 256, (E, H, I // 2), dtype=torch.uint8, device=dev, generator=g)
        sfu = _sf(E * I * H // 16, g)
        sfd = _sf(E * H * I // 16, g)
        gu = torch.rand(E, device=dev, generator=g) * 1e-3 + 1e-4
        gd = torch.rand(E, device=dev, generator=g) * 1e-3 + 1e-4
        y = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
        ws = torch.empty(metis.metis_workspace_size(metis.METIS_OP_MOE_NVFP4, T, I, H, k, E),
                         dtype=torch.uint8, device=dev)
        call = lambda: metis.metis_moe_nvfp4_grouped_gemm(x, ids, w, wu, sfu, gu, wd, sfd, gd, y, ws)
    elif a.op == "bf16":
        M, N, K = a.dims
        x = torch.randn(M, K, device=dev, generator=g).to(torch.bfloat16)
        wb = (torch.randn(N, K, device=dev, generator=g) * 0.03).to(torch.bfloat16)
        y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        call = lambda: metis.metis_bf16_gemm(x, wb, y)
    elif a.op == "gemm4":
        M, N, K = a.dims
        Mp = (M + 127) // 128 * 128
        qa = torch.randint(0, 256, (Mp, K // 2), dtype=torch.uint8, device=dev, generator=g)
        sa = _sf(Mp * K // 16, g)
        ga = torch.rand(M, device=dev, generator=g) + 0.5
        qb = torch.randint(0, 256, (N, K // 2), dtype=torch.uint8, device=dev, generator=g)
        sb = _sf(N * K // 16, g)
        gb = torch.ones(1, device=dev)
        y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        call = lambda: metis.metis_nvfp4_gemm(qa, sa, ga, qb, sb, gb, y)
    elif a.op in ("gemm", "fused"):
        M, N, K = a.dims
        x = torch.randn(M, K, device=dev, generator=g).to(torch.bfloat16)
        b = _codes(N, K, g)
        sb = torch.rand(N, device=dev, generator=g) + 0.5
        s = torch.empty(M, device=dev)
        y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        if a.op == "gemm":
            xq = torch.empty(M, K, dtype=torch.uint8, device=dev)
            metis.metis_quant_fp8_per_token(x, xq, s)
            call = lambda: metis.metis_fp8_gemm(xq, metis.METIS_A_E4M3, s, b, sb, y)
        else:
            ws = torch.empty(metis.metis_workspace_size(metis.METIS_OP_FP8_GEMM_FUSED, M, N, K, 0, 0),
                             dtype=torch.uint8, device=dev)
            call = lambda: metis.metis_fp8_gemm(x, metis.METIS_A_BF16, s, b, sb, y, workspace=ws)
    elif a.op in ("w16", "w16w"):
        M, N, K = a.dims
        x = torch.randn(M, K, device=dev, generator=g).to(torch.bfloat16)
        wq = _codes(N, K, g)
        sw = torch.rand(N, device=dev, generator=g) * 1e-3
        y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        if a.op == "w16":
            call = lambda: metis.metis_w8a16_gemm(x, wq, sw, y)
        else:  # weights widened into a workspace, then the BF16 CTA-pair GEMM
            ws = torch.empty(metis.metis_workspace_size(metis.METIS_OP_W8A16_WIDENED, M, N, K),
                             dtype=torch.uint8, device=dev)
            call = lambda: metis.metis_w8a16_gemm_widened(x, wq, sw, y, ws)
    elif a.op == "decode":
        (M,) = a.dims
        N, K = 14336, 4096
        x = torch.randn(M, K, device=dev, generator=g).to(torch.bfloat16)
        ws = [_codes(N, K, g) for _ in range(4)]  # 235 MB: larger than L2
        sw = torch.rand(N, device=dev, generator=g) * 1e-3
        y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        i = [0]

        def call():
            i[0] = (i[0] + 1) % 4
            metis.metis_w8a16_gemm(x, ws[i[0]], sw, y)
    else:
        M, K = a.dims
        x = torch.randn(M, K, device=dev, generator=g).to(torch.bfloat16)
        xq = torch.empty(M, K, dtype=torch.uint8, device=dev)
        s = torch.empty(M, device=dev)
        call = lambda: metis.metis_quant_fp8_per_token(x, xq, s)
    for _ in range(a.calls):
        call()
    torch.cuda.synchronize()
    rc = metis.metis_check_device_status()
    print(f"{a.op} {a.dims}: {a.calls} calls, device status {rc}")
    return 0 if rc == 0 else 1


if __name__ == "__main__":
    sys.exit(main())

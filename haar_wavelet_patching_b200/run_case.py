"""Run one operation of the library on a random workload, for profiling and timing.

    python -m haar_wavelet_patching_b200.run_case --op haar_inv --shape 1,3,33,704,1280 --dtype bf16 --iters 3
    python -m haar_wavelet_patching_b200.run_case --op fsq_encode --shape 48,16,56320 --iters 3
    python -m haar_wavelet_patching_b200.run_case --op haar_fwd_padded --shape 1,3,120,720,1280 --ms 16 --mt 8

Inputs are random tensors made on the device by torch (their values do not
change the kernels' work).  Prints the mean CUDA-event time per launch and the
algorithmic GB/s.
"""
import argparse

import torch

import haar_wavelet_patching_b200 as hwp


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--op", required=True, choices=("haar_fwd", "haar_inv", "haar_fwd_adjoint", "haar_inv_adjoint",
                                                     "haar_fwd_single", "haar_inv_single", "haar_fwd_channels_last",
                                                     "haar_fwd_padded", "haar_inv_cropped", "haar_fwd_chunk",
                                                     "haar_inv_chunk", "fsq_encode", "fsq_decode",
                                                     "fsq_encode_backward", "fsq_decode_backward",
                                                     "conv_spatial", "conv_temporal", "conv_factorized",
                                                     "patch_embed", "step"))
    ap.add_argument("--shape", required=True,
                    help="B,C,T,H,W for haar ops and step; B,C,S for fsq ops; B,T,h,w,Cin,Cmid,Cout for conv ops; "
                         "B,C,T,H,W,Cmid for patch_embed")
    ap.add_argument("--latent", default="64,16,56320",
                    help="step: B,C,S of the FSQ latent (the step is Haar fwd, Haar inv, FSQ encode, FSQ decode)")
    ap.add_argument("--dtype", default="bf16", choices=("bf16", "f32"))
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--codes", action="store_true", help="fsq_encode: also write the codes")
    ap.add_argument("--ms", type=int, default=4, help="padded ops: spatial multiple")
    ap.add_argument("--mt", type=int, default=4, help="padded ops: temporal multiple")
    ap.add_argument("--first", action="store_true", help="chunk ops: the first chunk (1 + 4k frames)")
    ap.add_argument("--flush", action="store_true",
                    help="flush L2 before each call (a 256 MB write and a 256 MB read, queued ahead of the call so "
                         "that no host time falls between the events) and time each call alone: for workloads that "
                         "fit in L2, and launches shorter than a call's host-side cost")
    a = ap.parse_args()
    shape = tuple(int(v) for v in a.shape.split(","))
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev).manual_seed(0)
    dt = torch.bfloat16 if a.dtype == "bf16" else torch.float32

    if a.op == "step":
        x = (torch.rand(shape, generator=g, device=dev) * 2 - 1).to(dt)
        y = torch.empty(hwp.haar_coeff_shape(*shape), dtype=dt, device=dev)
        xr = torch.empty_like(x)
        L = tuple(int(v) for v in a.latent.split(","))
        u = torch.randn(L, generator=g, device=dev)
        w = torch.randn(6, L[1], generator=g, device=dev) / L[1] ** 0.5
        idx = torch.empty(L[0], L[2], dtype=torch.int32, device=dev)
        ur = torch.empty_like(u)

        def run():
            hwp.tok_haar_fwd(x, y)
            hwp.tok_haar_inv(y, xr)
            hwp.tok_fsq_encode(u, w, idx)
            hwp.tok_fsq_decode(idx, w, ur)
        nbytes = 2 * (x.numel() + y.numel()) * x.element_size() + 2 * (u.numel() + idx.numel()) * 4
    elif a.op == "patch_embed":
        B, C, T, H, W, Cmid = shape
        bf = torch.bfloat16
        x = (torch.rand((B, C, T, H, W), generator=g, device=dev) * 2 - 1).to(bf)
        ws = (torch.randn((Cmid, 3, 3, 64 * C), generator=g, device=dev) * (9 * 64 * C) ** -0.5).to(bf)
        wp = hwp.patch_embed_pack_weights(ws)
        y = torch.empty((B, hwp.latent_frames(T), H // 4, W // 4, Cmid), dtype=bf, device=dev)
        run = lambda: hwp.tok_patch_embed_spatial(x, wp, y)  # noqa: E731
        flops = 2 * y.numel() // Cmid * Cmid * 9 * 64 * C
        nbytes = (x.numel() + y.numel()) * 2
    elif a.op.startswith("conv"):
        B, T, h, w, Cin, Cmid, Cout = shape
        bf = torch.bfloat16
        x = (torch.randn((B, T, h, w, Cin), generator=g, device=dev) * 0.5).to(bf)
        ws = (torch.randn((Cmid, 3, 3, Cin), generator=g, device=dev) * (9 * Cin) ** -0.5).to(bf)
        wt = (torch.randn((Cout, 3, Cmid), generator=g, device=dev) * (3 * Cmid) ** -0.5).to(bf)
        mid = torch.empty((B, T, h, w, Cmid), dtype=bf, device=dev)
        y = torch.empty((B, T, h, w, Cout), dtype=bf, device=dev)
        pos = B * T * h * w
        if a.op == "conv_spatial":
            run = lambda: hwp.tok_conv_spatial(x, ws, mid)  # noqa: E731
            flops, nbytes = 2 * pos * Cmid * 9 * Cin, (x.numel() + mid.numel() + ws.numel()) * 2
        elif a.op == "conv_temporal":
            run = lambda: hwp.tok_conv_temporal_causal(mid, wt, y)  # noqa: E731
            flops, nbytes = 2 * pos * Cout * 3 * Cmid, (mid.numel() + y.numel() + wt.numel()) * 2
        else:
            run = lambda: hwp.tok_conv_factorized(x, ws, wt, mid, y)  # noqa: E731
            flops = 2 * pos * (Cmid * 9 * Cin + Cout * 3 * Cmid)
            nbytes = (x.numel() + 2 * mid.numel() + y.numel() + ws.numel() + wt.numel()) * 2
    elif a.op == "haar_fwd_channels_last":
        x = (torch.rand(shape, generator=g, device=dev) * 2 - 1).to(dt)
        y = torch.empty(hwp.channels_last_shape(*shape), dtype=dt, device=dev)
        run = lambda: hwp.tok_haar_fwd_channels_last(x, y)  # noqa: E731
        nbytes = (x.numel() + y.numel()) * x.element_size()
    elif a.op in ("haar_fwd_single", "haar_inv_single"):
        x = (torch.rand(shape, generator=g, device=dev) * 2 - 1).to(dt)
        y = (torch.rand(hwp.single_coeff_shape(*shape), generator=g, device=dev) * 2 - 1).to(dt)
        run = (lambda: hwp.tok_haar_fwd_single(x, y)) if a.op == "haar_fwd_single" else \
            (lambda: hwp.tok_haar_inv_single(y, x))
        nbytes = (x.numel() + y.numel()) * x.element_size()
    elif a.op in ("haar_fwd_padded", "haar_inv_cropped", "haar_fwd_chunk", "haar_inv_chunk"):
        B, C, T, H, W = shape
        x = (torch.rand(shape, generator=g, device=dev) * 2 - 1).to(dt)
        if a.op.endswith(("padded", "cropped")):
            yshape = hwp.padded_coeff_shape(B, C, T, H, W, a.ms, a.mt)
        else:
            yshape = hwp.chunk_coeff_shape(B, C, T, H, W, a.first)
        y = (torch.rand(yshape, generator=g, device=dev) * 2 - 1).to(dt)
        run = {"haar_fwd_padded": lambda: hwp.tok_haar_fwd_padded(x, y, a.ms, a.mt),
               "haar_inv_cropped": lambda: hwp.tok_haar_inv_cropped(y, x, a.ms, a.mt),
               "haar_fwd_chunk": lambda: hwp.tok_haar_fwd_chunk(x, y, a.first),
               "haar_inv_chunk": lambda: hwp.tok_haar_inv_chunk(y, x, a.first)}[a.op]
        nbytes = (x.numel() + y.numel()) * x.element_size()
    elif a.op.startswith("haar"):
        B, C, T, H, W = shape
        x = (torch.rand(shape, generator=g, device=dev) * 2 - 1).to(dt)
        y = torch.empty(hwp.haar_coeff_shape(*shape), dtype=dt, device=dev)
        if a.op in ("haar_inv", "haar_fwd_adjoint"):
            y.copy_((torch.rand(y.shape, generator=g, device=dev) * 2 - 1).to(dt))
        run = {"haar_fwd": lambda: hwp.tok_haar_fwd(x, y), "haar_inv": lambda: hwp.tok_haar_inv(y, x),
               "haar_fwd_adjoint": lambda: hwp.tok_haar_fwd_adjoint(y, x),
               "haar_inv_adjoint": lambda: hwp.tok_haar_inv_adjoint(x, y)}[a.op]
        nbytes = (x.numel() + y.numel()) * x.element_size()
    else:
        B, C, S = shape
        w = torch.randn(6, C, generator=g, device=dev) / C ** 0.5
        u = torch.randn(shape, generator=g, device=dev)
        idx = torch.randint(0, hwp.FSQ_CODEBOOK, (B, S), generator=g, device=dev, dtype=torch.int32)
        codes = torch.empty(B, 6, S, device=dev) if a.codes else None
        if a.op == "fsq_encode":
            run = lambda: hwp.tok_fsq_encode(u, w, idx, codes)  # noqa: E731
            nbytes = (u.numel() + idx.numel() + (codes.numel() if codes is not None else 0)) * 4
        elif a.op == "fsq_decode":
            run = lambda: hwp.tok_fsq_decode(idx, w, u)  # noqa: E731
            nbytes = (u.numel() + idx.numel()) * 4
        else:
            ws = torch.empty(max(hwp.fsq_backward_workspace_size(B, C, S), 1), dtype=torch.uint8, device=dev)
            gw = torch.empty_like(w)
            g6 = torch.randn(B, 6, S, generator=g, device=dev)
            gout = torch.empty_like(u)
            if a.op == "fsq_encode_backward":
                run = lambda: hwp.tok_fsq_encode_backward(u, w, g6, gout, gw, ws)  # noqa: E731
                nbytes = (2 * u.numel() + g6.numel()) * 4
            else:
                run = lambda: hwp.tok_fsq_decode_backward(idx, w, u, g6, gw, ws)  # noqa: E731
                nbytes = (u.numel() + idx.numel() + g6.numel()) * 4

    run()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if a.flush:
        bufs = [torch.empty(256 << 20, dtype=torch.uint8, device=dev) for _ in range(2)]
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(a.iters)]
        for b0, b1 in evs:
            bufs[0].zero_()
            bufs[1].sum()
            b0.record()
            run()
            b1.record()
        torch.cuda.synchronize()
        ms = sum(b0.elapsed_time(b1) for b0, b1 in evs) / a.iters
    else:
        e0.record()
        for _ in range(a.iters):
            run()
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / a.iters
    extra = f", {flops / ms / 1e9:.1f} TFLOP/s" if a.op.startswith(("conv", "patch")) else ""
    print(f"{a.op} {shape} {a.dtype}: {ms * 1e3:.1f} us per launch, {nbytes / ms / 1e6:.1f} GB/s{extra}")


if __name__ == "__main__":
    main()

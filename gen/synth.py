"""Seeded synthetic Q/K/V in raster order [B, N, heads, head_dim], bf16.

Token order: the prefix segments first (each padded with trailing pad
tokens to a whole number of 64-token blocks), then the video grid in
(t, y, x) raster order, so video token (t, y, x) sits at P + (t*H + y)*W + x.

Value recipe per tensor (Q, K, V drawn from independent seeded streams):
  video tokens   x = 0.5*N(0,1) + sin(2*pi*(kt*t/T + ky*y/H + kx*x/W) + phi)
                 with (kt, ky, kx) in {0,1,2}^3 drawn per (head, channel) and
                 phi ~ U[0, 2*pi) drawn per (batch, head, channel): a smooth
                 low-frequency field, so block means carry structure;
  moving blobs   (optional, Q and K only) Gaussian blobs of sigma 4 tokens and
                 amplitude 2, each moving 2 tokens per frame on the (periodic)
                 frame, added with a random sign per (head, channel);
  prefix tokens  i.i.d. 0.5*N(0,1);
  pad tokens     a constant fill (1e4 in correctness runs, so that any pad
                 leaking into a result is visible; 0 in timing runs).
The seeds used are base + workload index; 42001 is the seed of the H100 runs
in the Prism speed ablation (oh-my-gpu.com, section on the dynamic-block
speed).
"""
import math

import torch

from .configs import derived_sizes


def _gen(seed, stream, device):
    g = torch.Generator(device=device)
    g.manual_seed((int(seed) * 1_000_003 + int(stream) * 7_919) % (2 ** 63 - 1))
    return g


def _video_coords(cfg, device):
    T, H, W = cfg["T"], cfg["H"], cfg["W"]
    t = torch.arange(T, device=device, dtype=torch.float32)
    y = torch.arange(H, device=device, dtype=torch.float32)
    x = torch.arange(W, device=device, dtype=torch.float32)
    tt, yy, xx = torch.meshgrid(t, y, x, indexing="ij")
    return tt.reshape(-1), yy.reshape(-1), xx.reshape(-1)


def _blob_field(cfg, n_blobs, g, device):
    """[T*H*W] sum of moving Gaussian blobs on the periodic frame."""
    T, H, W = cfg["T"], cfg["H"], cfg["W"]
    tt, yy, xx = _video_coords(cfg, device)
    field = torch.zeros_like(tt)
    sigma, amp, speed = 4.0, 2.0, 2.0
    for _ in range(n_blobs):
        y0 = torch.rand((), generator=g, device=device) * H
        x0 = torch.rand((), generator=g, device=device) * W
        ang = torch.rand((), generator=g, device=device) * (2 * math.pi)
        cy = y0 + speed * torch.sin(ang) * tt
        cx = x0 + speed * torch.cos(ang) * tt
        dy = torch.remainder(yy - cy + H / 2, H) - H / 2
        dx = torch.remainder(xx - cx + W / 2, W) - W / 2
        field = field + amp * torch.exp(-(dy * dy + dx * dx) / (2 * sigma * sigma))
    return field


def make_tensor(cfg, seed, tensor_id, pad_fill=1e4, device="cpu"):
    """One of Q (0), K (1), V (2) as bf16 [B, N, heads, head_dim]."""
    B, h, d = cfg["B"], cfg["heads"], cfg["head_dim"]
    sz = derived_sizes(cfg)
    N, P, Nv = sz["N"], sz["P"], sz["Nv"]
    g = _gen(seed, tensor_id, device)
    out = torch.empty((B, N, h, d), dtype=torch.bfloat16, device=device)

    kvec = torch.randint(0, 3, (3, h, d), generator=g, device=device).float()
    phi = torch.rand((B, h, d), generator=g, device=device) * (2 * math.pi)
    tt, yy, xx = _video_coords(cfg, device)
    base = 2 * math.pi * (tt[:, None, None] * kvec[0] / cfg["T"]
                          + yy[:, None, None] * kvec[1] / cfg["H"]
                          + xx[:, None, None] * kvec[2] / cfg["W"])  # [Nv,h,d]
    blob = None
    # moving objects go into Q and K (what block pooling and the dynamic
    # shape rule look at); V keeps the base recipe so that outputs stay in
    # the few-unit range where a bf16 result is accurate to ~1e-2 absolute
    if cfg.get("blobs", 0) and tensor_id in (0, 1):
        gb = _gen(seed, 100 + tensor_id, device)
        field = _blob_field(cfg, cfg["blobs"], gb, device)
        sign = torch.randint(0, 2, (h, d), generator=gb, device=device).float() * 2 - 1
        blob = field[:, None, None] * sign
    for b in range(B):
        noise = torch.randn((Nv, h, d), generator=g, device=device) * 0.5
        vid = noise + torch.sin(base + phi[b])
        if blob is not None:
            vid = vid + blob
        out[b, P:] = vid.to(torch.bfloat16)
        del noise, vid
    if P:
        out[:, :P] = (torch.randn((B, P, h, d), generator=g, device=device) * 0.5
                      ).to(torch.bfloat16)

    # pad tokens: trailing slots of each prefix segment, and video tokens
    # outside the valid extents of the grid
    off = 0
    for n in cfg["prefix"]:
        padded = ((n + 63) // 64) * 64
        if padded > n:
            out[:, off + n:off + padded] = pad_fill
        off += padded
    T, H, W = cfg["T"], cfg["H"], cfg["W"]
    if (cfg["T_valid"], cfg["H_valid"], cfg["W_valid"]) != (T, H, W):
        vid = out[:, P:].view(B, T, H, W, h, d)
        vid[:, cfg["T_valid"]:] = pad_fill
        vid[:, :, cfg["H_valid"]:] = pad_fill
        vid[:, :, :, cfg["W_valid"]:] = pad_fill
    return out


def make_qkv(cfg, seed, pad_fill=1e4, device="cpu"):
    return tuple(make_tensor(cfg, seed, i, pad_fill, device) for i in range(3))


def make_gate(heads, head_dim, seed, spread=0.5, device="cpu"):
    """Synthetic gate matrices fp32 [heads, d, d] standing in for trained
    to_gate_compress weights (none are available): identity plus seeded
    Gaussian entries of standard deviation spread/sqrt(d), so the gated
    selection differs from the plain pooled score but keeps its structure."""
    g = _gen(seed, 50, device)
    eye = torch.eye(head_dim, device=device).expand(heads, head_dim, head_dim)
    noise = torch.randn((heads, head_dim, head_dim), generator=g, device=device)
    return (eye + noise * (spread / math.sqrt(head_dim))).float().contiguous()


def layer_keep_schedule(n_layers=40, seed=42004, choices=(0.01, 0.03, 0.05, 0.10)):
    """Per-layer keep ratios drawn by seed from the 1/3/5/10 % menu that the
    "倍速で回した一晩" digest's layer controller chose from."""
    g = torch.Generator().manual_seed(seed)
    pick = torch.randint(0, len(choices), (n_layers,), generator=g)
    return [choices[i] for i in pick.tolist()]

"""Workload shapes for block-sparse video attention.

Each entry is a plain dict describing one attention call: batch, heads,
head_dim, the padded token grid T x H x W with its valid extents, the
conditioning-prefix segment lengths, the keep ratio of video key blocks and
the block mode (0 = fixed 4x4x4 tiles, 1 = per-8x8x8-region dynamic tiles).

Grid sizes follow the video workloads on the pages:
  * 720p, 121 frames -> a 32 x 48 x 80 token grid, 122,880 tokens
    (Prism/Kandinsky 6 speed ablation, oh-my-gpu.com, section on the
    quadratic attention cost);
  * sparsity 0.75 keeps 25 % of key blocks (same page, Prism section);
  * 1344 x 768 reference-conditioned clips with a text / reference-image /
    reference-audio prefix kept dense (Ref2VA VSA, pulmap.app, section on
    condition tokens);
  * keep ratios of 1, 3, 5, 10 % and the 7.93 / 6.64 % points of the
    below-10 % sweep (the "倍速で回した一晩" digest, section on going
    below 10 %).
"""
import copy

# keep ratios of the aggressive-sparsity sweep workload
SWEEP_KEEP_RATIOS = (0.25, 0.10, 0.0793, 0.0664, 0.05, 0.03, 0.01)

_BASE = dict(B=1, heads=24, head_dim=128, prefix=(), block_mode=0,
             dyn_tau=1.25, blobs=0)

CONFIGS = {
    # 8x16x16 grid, 2 heads of 64, 32 fixed blocks, keep 8 (sparsity 0.75)
    "tiny": dict(_BASE, B=1, heads=2, head_dim=64, T=8, H=16, W=16,
                 T_valid=8, H_valid=16, W_valid=16, keep_ratio=0.25),
    # 768x432 latent: 24x28x48 grid whose 28th row is padding
    "lowres": dict(_BASE, T=24, H=28, W=48, T_valid=24, H_valid=27,
                   W_valid=48, keep_ratio=0.25),
    # 720p 121-frame clip, CFG cond/uncond stacked as B=2
    "720p": dict(_BASE, B=2, T=32, H=48, W=80, T_valid=32, H_valid=48,
                 W_valid=80, keep_ratio=0.25),
    # same grid with dynamic per-region block shapes and moving objects; the
    # blob count is calibrated so that about 40 % of the 8x8x8 regions pick a
    # non-default shape at tau = 1.25 (64 blobs: 38 % for the K of batch 0)
    "720p_dyn": dict(_BASE, B=2, T=32, H=48, W=80, T_valid=32, H_valid=48,
                     W_valid=80, keep_ratio=0.25, block_mode=1, blobs=64),
    # 1344x768 clip behind a 512 text + 2048 image + 256 audio prefix
    "ref_prefix": dict(_BASE, T=32, H=48, W=84, T_valid=32, H_valid=48,
                       W_valid=84, prefix=(512, 2048, 256), keep_ratio=0.25),
    # 1152x640 aggressive-sparsity sweep grid (keep ratio set per run)
    "sweep": dict(_BASE, T=32, H=40, W=72, T_valid=32, H_valid=40,
                  W_valid=72, keep_ratio=0.10),
}


def config(name, **overrides):
    """A deep copy of a named workload with fields overridden."""
    c = copy.deepcopy(CONFIGS[name])
    c.update(overrides)
    c["name"] = name
    return c


def derived_sizes(cfg):
    """Token and 64-token block counts of a workload (pure shape arithmetic)."""
    pre_pad = [((n + 63) // 64) * 64 for n in cfg["prefix"]]
    P = sum(pre_pad)
    Nv = cfg["T"] * cfg["H"] * cfg["W"]
    return dict(P=P, N=P + Nv, Nv=Nv, nbp=P // 64, nbv=Nv // 64,
                nb=(P + Nv) // 64)

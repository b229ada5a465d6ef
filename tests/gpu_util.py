"""Helpers for the GPU tests: moving seeded numpy inputs to the device and back."""
import numpy as np


def dev(a, dtype=None):
    import torch

    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:  # bf16 bit patterns
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    t = torch.from_numpy(a).cuda()
    return t if dtype is None else t.to(dtype)


def host(t):
    import torch

    t = t.detach()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def make_cache(fp4, scale, n_blocks, block, idx_key=None, idx_dtype=0, scale_fmt=0, idx_key_scale=None):
    """Device cache from numpy planes (idx_key as raw bytes [B, cap, key_bytes]; MXFP4 keys:
    codes [B, cap, dI/2] and idx_key_scale [B, cap, dI/32])."""
    import torch

    import fp4_kv_cache_csa_b200 as csa

    ik = None
    if idx_key is not None:
        ik = dev(idx_key)
        if idx_dtype == 0:
            ik = ik.view(torch.bfloat16)
    return csa.Cache(fp4=dev(fp4), scale=dev(scale), n_blocks=dev(np.asarray(n_blocks, np.int32)), block=block,
                     idx_key=ik, idx_dtype=idx_dtype, status=torch.zeros(1, dtype=torch.int32, device="cuda"),
                     scale_fmt=scale_fmt, idx_key_scale=None if idx_key_scale is None else dev(idx_key_scale))

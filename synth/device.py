"""Device-side evaluation of the seeded generator (libsynth.so): returns torch
tensors on the current CUDA device.  Bits equal ``synth.bf16_at`` on the host.
No arithmetic of the attention method lives here."""
from __future__ import annotations

import torch

from . import T_K, T_LATENT, T_V, device_lib, key, q_tensor


def _stream():
    return torch.cuda.current_stream().cuda_stream


def fill_flat(out: torch.Tensor, seed: int, tensor: int) -> torch.Tensor:
    """out (bf16, contiguous) <- stream key(seed, tensor) at flat indices."""
    st = device_lib().synth_fill_flat(out.data_ptr(), out.numel(), key(seed, tensor), _stream())
    if st != 0:
        raise RuntimeError(f"synth_fill_flat failed ({st})")
    return out


def q(seed: int, B: int, hq: int, dk: int, step: int = 0, device="cuda") -> torch.Tensor:
    t = torch.empty((B, hq, dk), dtype=torch.bfloat16, device=device)
    return fill_flat(t, seed, q_tensor(step))


def kv_rows(seed: int, tensor: int, req: torch.Tensor, pos: torch.Tensor, hkv: int, w: int) -> torch.Tensor:
    """Rows [n][hkv][w] (bf16) of the K / V / latent stream for (req[i], pos[i])."""
    n = pos.numel()
    out = torch.empty((n, hkv, w), dtype=torch.bfloat16, device=pos.device)
    if n:
        st = device_lib().synth_fill_kv_rows(out.data_ptr(), n, req.data_ptr(), pos.data_ptr(), hkv, w,
                                             key(seed, tensor), _stream())
        if st != 0:
            raise RuntimeError(f"synth_fill_kv_rows failed ({st})")
    return out


def gqa_rows(seed: int, req, pos, hkv: int, d: int):
    return kv_rows(seed, T_K, req, pos, hkv, d), kv_rows(seed, T_V, req, pos, hkv, d)


def latent_rows(seed: int, req, pos):
    return kv_rows(seed, T_LATENT, req, pos, 1, 576).view(-1, 576)

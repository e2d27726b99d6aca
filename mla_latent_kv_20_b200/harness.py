"""Device-side setup helpers built on the public API: torch buffers, cache fill, one decode step.

These only allocate device memory (PyTorch) and call the C ABI through the binding; all
arithmetic happens in the library's kernels.
"""
from __future__ import annotations

import math

import numpy as np
import torch

from . import (D_HEAD, D_LATENT, D_ROPE, D_ROW, N_HEADS, PAGE_SIZE, CacheDesc, absorb_q, cache_append,
               cache_append_fp8, contiguous_desc, decode_attn, decode_attn_fp8, decode_workspace_size, paged_desc,
               unabsorb_v)

SCALE = 1.0 / math.sqrt(D_HEAD + D_ROPE)


def bf16_tensor(bits: np.ndarray, device="cuda") -> torch.Tensor:
    """uint16 bf16 bit patterns -> a bf16 torch tensor on `device`."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.to(device)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


class Cache:
    """One layer's latent cache (contiguous or paged) plus its descriptor."""

    def __init__(self, seq_lens, paged: bool, block_table: np.ndarray | None = None, num_blocks: int = 0,
                 max_seq_len: int | None = None, device="cuda", fill_value: float | None = 0.0):
        seq_lens = np.asarray(seq_lens, dtype=np.int32)
        self.seq_lens_np = seq_lens
        self.paged = paged
        B = len(seq_lens)
        if paged:
            assert block_table is not None
            self.block_table = torch.from_numpy(np.ascontiguousarray(block_table, dtype=np.int32)).to(device)
            self.desc = paged_desc(B, block_table.shape[1], num_blocks)
            rows = num_blocks * PAGE_SIZE
        else:
            L = int(max_seq_len if max_seq_len is not None else max(int(seq_lens.max()), 1))
            self.block_table = None
            self.desc = contiguous_desc(B, L)
            rows = B * L
        if fill_value is None:
            self.data = torch.empty((rows, D_ROW), dtype=torch.bfloat16, device=device)
        else:
            self.data = torch.full((rows, D_ROW), fill_value, dtype=torch.bfloat16, device=device)
        self.seq_lens = torch.from_numpy(seq_lens).to(device)

    def capacity(self) -> int:
        d = self.desc
        return d.max_seq_len if d.page_size == 0 else d.max_blocks_per_seq * PAGE_SIZE

    def fill(self, c_list, kr_list, rope_base: float = 10000.0, stream=None):
        """Append every token of every sequence (token t at position t) with one library call."""
        seq_ids = np.concatenate([np.full(len(c), i, np.int32) for i, c in enumerate(c_list)])
        pos = np.concatenate([np.arange(len(c), dtype=np.int32) for c in c_list])
        if len(pos) == 0:
            return
        c = bf16_tensor(np.concatenate(c_list, axis=0), self.data.device)
        kr = bf16_tensor(np.concatenate(kr_list, axis=0), self.data.device)
        cache_append(c, kr, torch.from_numpy(pos).to(self.data.device), self.data, self.desc,
                     seq_ids=torch.from_numpy(seq_ids).to(self.data.device), block_table=self.block_table,
                     rope_base=rope_base, stream=stream)

    def row_index(self, b: int, t: int) -> int:
        if not self.paged:
            return b * self.desc.max_seq_len + t
        return int(self.block_table[b, t // PAGE_SIZE].item()) * PAGE_SIZE + t % PAGE_SIZE


class Fp8Cache(Cache):
    """One layer's FP8 latent cache: E4M3 codes [rows, 576] and E8M0 row scales [rows], same geometry
    (contiguous rows padded to a multiple of 16 per sequence, or 64-token pages)."""

    def __init__(self, seq_lens, paged: bool, block_table: np.ndarray | None = None, num_blocks: int = 0,
                 max_seq_len: int | None = None, device="cuda", fill_byte: int | None = 0):
        seq_lens = np.asarray(seq_lens, dtype=np.int32)
        if not paged and max_seq_len is None:
            max_seq_len = (max(int(seq_lens.max()), 1) + 15) // 16 * 16
        super().__init__(seq_lens, paged, block_table, num_blocks, max_seq_len, device, fill_value=None)
        rows = self.data.shape[0]
        self.data = (torch.empty if fill_byte is None else torch.zeros)((rows, D_ROW), dtype=torch.uint8,
                                                                         device=device)
        self.scales = (torch.empty if fill_byte is None else torch.zeros)((rows,), dtype=torch.uint8, device=device)
        if fill_byte:
            self.data.fill_(fill_byte)
            self.scales.fill_(fill_byte)

    def fill(self, c_list, kr_list, rope_base: float = 10000.0, stream=None):
        seq_ids = np.concatenate([np.full(len(c), i, np.int32) for i, c in enumerate(c_list)])
        pos = np.concatenate([np.arange(len(c), dtype=np.int32) for c in c_list])
        if len(pos) == 0:
            return
        dev = self.data.device
        c = bf16_tensor(np.concatenate(c_list, axis=0), dev)
        kr = bf16_tensor(np.concatenate(kr_list, axis=0), dev)
        cache_append_fp8(c, kr, torch.from_numpy(pos).to(dev), self.data, self.scales, self.desc,
                         seq_ids=torch.from_numpy(seq_ids).to(dev), block_table=self.block_table,
                         rope_base=rope_base, stream=stream)


def decode_fp8(q_full: torch.Tensor, cache: Fp8Cache, *, num_splits: int = 0, scale: float = SCALE, stream=None):
    B = q_full.shape[0]
    out_lat = torch.empty((B, N_HEADS, D_LATENT), dtype=torch.bfloat16, device=q_full.device)
    lse = torch.empty((B, N_HEADS), dtype=torch.float32, device=q_full.device)
    nbytes = decode_workspace_size(B, cache.capacity(), num_splits)
    workspace = torch.empty((max(nbytes, 16),), dtype=torch.uint8, device=q_full.device)
    decode_attn_fp8(q_full, cache.data, cache.scales, cache.seq_lens, cache.desc, workspace, out_lat, lse=lse,
                    block_table=cache.block_table, softmax_scale=scale, num_splits=num_splits, stream=stream)
    return out_lat, lse


def decode(q_full: torch.Tensor, cache: Cache, *, num_splits: int = 0, with_lse: bool = True,
           scale: float = SCALE, workspace: torch.Tensor | None = None, stream=None):
    B = q_full.shape[0]
    out_lat = torch.empty((B, N_HEADS, D_LATENT), dtype=torch.bfloat16, device=q_full.device)
    lse = torch.empty((B, N_HEADS), dtype=torch.float32, device=q_full.device) if with_lse else None
    if workspace is None:
        nbytes = decode_workspace_size(B, cache.capacity(), num_splits)
        workspace = torch.empty((max(nbytes, 16),), dtype=torch.uint8, device=q_full.device)
    decode_attn(q_full, cache.data, cache.seq_lens, cache.desc, workspace, out_lat, lse=lse,
                block_table=cache.block_table, softmax_scale=scale, num_splits=num_splits, stream=stream)
    return out_lat, lse


def decode_step(q_nope, q_pe, w_uk, w_uv, cache: Cache, *, q_pos=None, num_splits: int = 0, stream=None):
    """absorb -> decode attention -> un-absorb; returns (out, out_lat, lse, q_full)."""
    B = q_nope.shape[0]
    q_full = torch.empty((B, N_HEADS, D_ROW), dtype=torch.bfloat16, device=q_nope.device)
    absorb_q(q_nope, q_pe, w_uk, q_full, q_pos=q_pos, stream=stream)
    out_lat, lse = decode(q_full, cache, num_splits=num_splits, stream=stream)
    out = torch.empty((B, N_HEADS, D_HEAD), dtype=torch.bfloat16, device=q_nope.device)
    unabsorb_v(out_lat, w_uv, out, stream=stream)
    return out, out_lat, lse, q_full

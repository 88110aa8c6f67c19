"""Context-parallel prefill: one long sequence cut into consecutive parts, one
part per rank (one process per GPU, ``torch.distributed`` over NCCL).

The Qwen3.5 family is built for long contexts ("Qwen/Qwen3.5-9B", config
table: max_position_embeddings 262144; "Qwen3.5-397B-A17B", specification
table: 256K tokens natively).  The gated delta rule is linear in its state
(S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T: "Qwen (text &
vision-language)", Architecture notes), so over a part the state after it is
an affine function of the state before it, S_after = S_before M + R.  A rank
therefore needs nothing from the other ranks but

  1. the last three raw inputs before its part (the conv history; they may
     reach back over several short parts), gathered from every rank's tail;
  2. the start state of its part, the fold of the maps (M, R) of all earlier
     parts from the sequence's initial state.

Per rank: exchange the tails (3 x Cc values each), compute the map of the own
part (``gdn_prefill_state_map``), all-gather the maps (2 Hv d^2 fp32 each),
fold the earlier ones (``gdn_state_fold``) and run ``gdn_prefill`` on the own
part from that start state.  The last rank's final state is the sequence's;
it is broadcast to every rank.

The arithmetic runs in the library's kernels; this module only moves tensors.
The compute calls are an object with ``state_map``, ``fold`` and ``prefill``
methods, :class:`LibraryCompute` by default, so that the exchange logic can be
exercised on CPU ranks with another implementation of the same three calls.
"""
from __future__ import annotations

from dataclasses import dataclass, replace
from typing import List, Optional, Sequence

import torch
import torch.distributed as dist

from . import api


@dataclass
class PartResult:
    out: torch.Tensor          # [T_part, Hv, d] this rank's outputs
    final_state: torch.Tensor  # [1, Hv, d, d] the state after the whole sequence (every rank)
    start_state: torch.Tensor  # [1, Hv, d, d] the state before this rank's part
    conv_history: torch.Tensor  # [1, Cc, 3] the raw inputs before this rank's part


class LibraryCompute:
    """The three calls on the CUDA library (parts are ``api.DevicePrefill``).

    A part's workspace is kept from its map to its prefill, which then skips
    the conv and the key-side kernel (``reuse_workspace``)."""

    def __init__(self, segments: int = 0, reuse: bool = True):
        self.segments = segments
        self.reuse = reuse
        self._bufs = {}

    @staticmethod
    def _key(part):
        return (part.mixed_qkv.data_ptr(), part.T)

    def state_map(self, part: api.DevicePrefill) -> torch.Tensor:
        bufs = api.PrefillBuffers(part)
        self._bufs[self._key(part)] = bufs
        return api.state_map(part, bufs, segments=self.segments)

    def fold(self, maps: torch.Tensor, S_first: Optional[torch.Tensor], part: api.DevicePrefill) -> torch.Tensor:
        return api.state_fold(maps, S_first, part.Hk, part.Hv, part.d)

    def prefill(self, part: api.DevicePrefill):
        bufs = self._bufs.pop(self._key(part), None)
        if self.reuse and bufs is not None and part.T > 0:
            r = api.prefill(part, bufs=bufs, reuse_workspace=True)
        else:
            r = api.prefill(part)
        return r.out.clone(), r.final_state.clone()


def conv_history(h0: torch.Tensor, tails: torch.Tensor, lens: Sequence[int], r: int) -> torch.Tensor:
    """The last three raw inputs before part r, [Cc, 3] oldest first.

    h0: [Cc, 3] the sequence's own conv history (zeros for a fresh sequence);
    tails: [W, 3, Cc], part j's last min(3, lens[j]) raw rows at the end of
    tails[j]; lens: the parts' token counts."""
    hist = h0.t()
    for j in range(r):
        take = min(3, int(lens[j]))
        if take:
            hist = torch.cat([hist, tails[j, 3 - take:]], dim=0)[-3:]
    return hist.t().contiguous()


def _tail(x: torch.Tensor) -> torch.Tensor:
    """Last min(3, T) rows of x [T, Cc], right-aligned in a [3, Cc] block."""
    t = torch.zeros((3, x.shape[1]), dtype=x.dtype, device=x.device)
    take = min(3, x.shape[0])
    if take:
        t[3 - take:] = x[x.shape[0] - take:]
    return t


def prefill_context_parallel(part: api.DevicePrefill, group=None, compute=None,
                             initial_state: Optional[torch.Tensor] = None,
                             conv_state_in: Optional[torch.Tensor] = None) -> PartResult:
    """This rank's share of a context-parallel prefill of one sequence.

    part: this rank's consecutive tokens of the sequence (N = 1), rank order =
    token order.  initial_state [1, Hv, d, d] / conv_state_in [1, Cc, 3]: the
    sequence's own, the same on every rank (None: zeros); part.initial_state
    and part.conv_state_in are ignored.  Every rank calls this with its part;
    the collectives, in this order on every rank: an all-gather of the tails,
    one of the lengths, one of the maps, and a broadcast of the final state."""
    compute = compute or LibraryCompute()
    W = dist.get_world_size(group)
    r = dist.get_rank(group)
    x = part.mixed_qkv
    Cc = x.shape[1]
    # 1. conv histories: every part's tail and length
    tail_list = [torch.empty((3, Cc), dtype=x.dtype, device=x.device) for _ in range(W)]
    dist.all_gather(tail_list, _tail(x).contiguous(), group=group)
    tails = torch.stack(tail_list)
    len_list = [torch.empty((1,), dtype=torch.int64, device=x.device) for _ in range(W)]
    dist.all_gather(len_list, torch.tensor([x.shape[0]], dtype=torch.int64, device=x.device), group=group)
    lens = [int(v.item()) for v in len_list]
    h0 = (conv_state_in.reshape(Cc, 3) if conv_state_in is not None
          else torch.zeros((Cc, 3), dtype=x.dtype, device=x.device))
    hist = conv_history(h0, tails, lens, r).reshape(1, Cc, 3)
    me = replace(part, conv_state_in=hist, initial_state=None)
    # 2. the map of this part, gathered from every rank
    m = compute.state_map(me).contiguous()  # [1, Hv, 2, d, d]
    map_list = [torch.empty_like(m) for _ in range(W)]
    dist.all_gather(map_list, m, group=group)
    maps = torch.stack(map_list)
    # 3. the start state of this part, then the part itself
    S_start = compute.fold(maps[:r], initial_state, me)
    out, final = compute.prefill(replace(me, initial_state=S_start))
    # 4. the sequence's final state comes from the last rank
    final = final.contiguous()
    dist.broadcast(final, src=dist.get_global_rank(group, W - 1) if group is not None else W - 1, group=group)
    return PartResult(out=out, final_state=final, start_state=S_start, conv_history=hist)


def split_sequence(dp: api.DevicePrefill, lens: Sequence[int]) -> List[api.DevicePrefill]:
    """Cut a one-sequence prefill input into consecutive parts of the given
    token counts (each part's tensors freshly allocated)."""
    assert dp.N == 1 and sum(lens) == dp.T
    parts, t0 = [], 0
    for L in lens:
        sl = slice(t0, t0 + L)
        parts.append(replace(
            dp, N=1, T=L, cu_seqlens=torch.tensor([0, L], dtype=torch.int32, device=dp.cu_seqlens.device),
            mixed_qkv=dp.mixed_qkv[sl].clone(), a=dp.a[sl].clone(), b=dp.b[sl].clone(), z=dp.z[sl].clone(),
            initial_state=None, conv_state_in=None))
        t0 += L
    return parts


def prefill_parts_local(parts: List[api.DevicePrefill], compute=None,
                        initial_state: Optional[torch.Tensor] = None,
                        conv_state_in: Optional[torch.Tensor] = None) -> List[PartResult]:
    """The same computation for all parts in one process (no collectives):
    what the ranks of ``prefill_context_parallel`` compute together, for
    checking it on one device."""
    compute = compute or LibraryCompute()
    x0 = parts[0].mixed_qkv
    Cc = x0.shape[1]
    tails = torch.stack([_tail(p.mixed_qkv) for p in parts])
    lens = [p.mixed_qkv.shape[0] for p in parts]
    h0 = (conv_state_in.reshape(Cc, 3) if conv_state_in is not None
          else torch.zeros((Cc, 3), dtype=x0.dtype, device=x0.device))
    mes, maps = [], []
    for r, p in enumerate(parts):
        hist = conv_history(h0, tails, lens, r).reshape(1, Cc, 3)
        mes.append(replace(p, conv_state_in=hist, initial_state=None))
        maps.append(compute.state_map(mes[-1]).contiguous())
    maps_t = torch.stack(maps)
    res = []
    for r, me in enumerate(mes):
        S_start = compute.fold(maps_t[:r], initial_state, me)
        out, final = compute.prefill(replace(me, initial_state=S_start))
        res.append(PartResult(out=out, final_state=final, start_state=S_start, conv_history=me.conv_state_in))
    for rr in res:
        rr.final_state = res[-1].final_state
    return res

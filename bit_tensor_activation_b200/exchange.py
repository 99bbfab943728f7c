"""The hybrid wire exchanged between real tensor-parallel ranks, one process per GPU.

Page "Revolutionizing LLM Inference: The Power of Efficient Low-Bit Communication": each rank
quantizes its partial sum *before* the ranks synchronise (section "Combating Quantization Errors
with Tensor Parallelism"), the wire is exchanged, and the received tensors are converted back and
summed (section "The Hybrid Quantization Algorithm", bullet "Inference"), with "a range of
AllReduce algorithms" left open (section "Key Observations and Future Directions").  This module
puts libhq's per-rank calls around one exchange step of torch.distributed collectives (NCCL
between GPUs):

  ``allgather``       every rank all-gathers every rank's wire (codes + side) and reduces all T rows
                      itself (one exchange step; the reduction is done P times over)
  ``reduce_scatter``  the wire is split into P row blocks; rank j receives block j of every rank's
                      wire (all-to-all), reduces it, and the reduced bf16 blocks are all-gathered
  ``peer``            (``PeerAllReduce``) every rank packs into its own part of a symmetric-memory
                      allocation and reduces all P wires reading the peers' buffers in place over
                      NVLink/NVSwitch (hq_dequant_reduce_ranks): the exchange and the reduction are
                      one kernel, with a barrier on each side
  two-step            (``TwoStepAllReduce``) ``reduce_scatter``'s first step, then each reducer
                      quantizes its reduced block again with its own 4-bit grid and the step-2
                      wires are all-gathered and dequantized: the quantized reduce-scatter plus
                      re-quantized all-gather of the "Flash Communication" abstract

Every remote byte lands in this rank's own receive buffers before a kernel reads it.  The
collective helpers move bytes only (each buffer is sent as its uint8 view), so they run on CPU
tensors over gloo as well, which is how the multi-process plumbing is tested without GPUs.  The
reductions are the library's kernels; nothing here does arithmetic on the data.

Each collective runs in rank order, so the received stack [P][...] is in rank order and the
reduction over it is bitwise the single-GPU reduction of the same P partial sums (the rows of a
reduction are independent, so reducing a row block gives those rows of the whole).
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist

from . import (hq_calibrate, hq_dequant_reduce, hq_dequant_reduce_ranks, hq_quantize_pack, hq_select_topk)


# ---------------------------------------------------------------------------------------------
# Collectives on raw bytes (any dtype, any device the process group supports)
# ---------------------------------------------------------------------------------------------
def _bytes(t: torch.Tensor) -> torch.Tensor:
    return t.contiguous().view(-1).view(torch.uint8)


def allgather_stack(local: torch.Tensor, group=None) -> torch.Tensor:
    """[1, ...] on every rank -> [P, ...]: rank r's tensor at index r."""
    P = dist.get_world_size(group)
    if local.shape[0] != 1:
        raise ValueError("the local tensor's first dimension must be 1")
    out = torch.empty((P,) + tuple(local.shape[1:]), dtype=local.dtype, device=local.device)
    if local.numel():
        dist.all_gather_into_tensor(_bytes(out), _bytes(local), group=group)
    return out


def alltoall_blocks(send: torch.Tensor, group=None) -> torch.Tensor:
    """[P, ...] with block j meant for rank j -> [P, ...] with block s received from rank s."""
    P = dist.get_world_size(group)
    if send.shape[0] != P:
        raise ValueError(f"the first dimension must be the world size {P}")
    out = torch.empty_like(send)
    if send.numel():
        dist.all_to_all_single(_bytes(out), _bytes(send), group=group)
    return out


def allgather_rows(block: torch.Tensor, group=None) -> torch.Tensor:
    """[Tb, ...] row block j on rank j -> [P * Tb, ...] in rank order."""
    P = dist.get_world_size(group)
    out = torch.empty((P * block.shape[0],) + tuple(block.shape[1:]), dtype=block.dtype, device=block.device)
    if block.numel():
        dist.all_gather_into_tensor(_bytes(out), _bytes(block), group=group)
    return out


# ---------------------------------------------------------------------------------------------
# Parameters shared by the ranks
# ---------------------------------------------------------------------------------------------
@dataclass
class HybridParams:
    """The selection and every rank's 4-bit grid, the same on all ranks.

    keep_idx [k], rest_idx [H-k] int32; scale, inv_scale [P, H] float32; zero [P, H] uint8.
    Rank r quantizes with row r; a receiver dequantizes rank r's wire with row r.
    """

    keep_idx: torch.Tensor
    rest_idx: torch.Tensor
    scale: torch.Tensor
    inv_scale: torch.Tensor
    zero: torch.Tensor

    @property
    def P(self) -> int:
        return self.scale.shape[0]

    @property
    def H(self) -> int:
        return self.scale.shape[1]

    @property
    def k(self) -> int:
        return self.keep_idx.shape[0]

    def row(self, r: int) -> tuple[torch.Tensor, torch.Tensor]:
        return self.inv_scale[r:r + 1], self.zero[r:r + 1]


def calibrate_local(x_local: torch.Tensor, ema_min: torch.Tensor, ema_max: torch.Tensor, beta: float,
                    first_batch: bool, stream=None) -> None:
    """Bullet "Calibration": this rank's moving averages over its own partial sums [T, H]
    (hq_calibrate with P = 1; ema_min/ema_max are [1, H])."""
    hq_calibrate(x_local.unsqueeze(0), ema_min, ema_max, beta, first_batch, stream=stream)


def select_shared(ema_min: torch.Tensor, ema_max: torch.Tensor, k: int, group=None) -> HybridParams:
    """Bullet "Selection of High Precision Features": every rank's statistics [1, H] are
    all-gathered once (one exchange after calibration), and every rank runs the same selection
    over the [P, H] statistics, so all ranks hold the same kept set and all ranks' grids."""
    emin = allgather_stack(ema_min, group)
    emax = allgather_stack(ema_max, group)
    P, H = emin.shape
    dev = emin.device
    p = HybridParams(keep_idx=torch.empty(k, dtype=torch.int32, device=dev),
                     rest_idx=torch.empty(H - k, dtype=torch.int32, device=dev),
                     scale=torch.empty((P, H), dtype=torch.float32, device=dev),
                     inv_scale=torch.empty((P, H), dtype=torch.float32, device=dev),
                     zero=torch.empty((P, H), dtype=torch.uint8, device=dev))
    hq_select_topk(emin, emax, k, p.keep_idx, p.rest_idx, p.scale, p.inv_scale, p.zero)
    return p


# ---------------------------------------------------------------------------------------------
# The compressed all-reduce
# ---------------------------------------------------------------------------------------------
def _check_row_aligned(H: int) -> None:
    """A rank's row of the parameters is passed to the library on its own; zero rows (one byte per
    feature) start on a 16-byte boundary only when H is a multiple of 16."""
    if H % 16:
        raise ValueError(f"the per-rank calls need H % 16 == 0 (H = {H})")


class HybridAllReduce:
    """All-reduce of this rank's partial sum x [T, H] (bf16) through the hybrid wire.

    The three phases are separate methods so that a caller (or a test) can run them apart:
    ``pack`` (this rank's quantize-pack), ``exchange`` (the collectives) and ``reduce`` (the
    dequant-reduce of what arrived, then for ``reduce_scatter`` the all-gather of the reduced rows).
    """

    def __init__(self, params: HybridParams, T: int, rank: int, scheme: str = "allgather", group=None):
        if scheme not in ("allgather", "reduce_scatter"):
            raise ValueError(f"unknown scheme {scheme}")
        P, H, k = params.P, params.H, params.k
        _check_row_aligned(H)
        if scheme == "reduce_scatter" and T % P:
            raise ValueError(f"reduce_scatter needs T % P == 0 (T={T}, P={P})")
        self.p, self.T, self.rank, self.scheme, self.group = params, T, rank, scheme, group
        dev = params.scale.device
        W = (H - k) // 8
        if scheme == "allgather":
            self.codes = torch.empty((1, T, W), dtype=torch.int32, device=dev)
            self.side = torch.empty((1, k, T), dtype=torch.bfloat16, device=dev)
            self.inv, self.zero = params.row(rank)
        else:
            Tb = T // P
            self.codes = torch.empty((P, Tb, W), dtype=torch.int32, device=dev)
            self.side = torch.empty((P, k, Tb), dtype=torch.bfloat16, device=dev)
            # the row blocks of one rank's partial sum all use that rank's grid
            self.inv = params.inv_scale[rank:rank + 1].expand(P, H).contiguous()
            self.zero = params.zero[rank:rank + 1].expand(P, H).contiguous()

    def pack(self, x: torch.Tensor, stream=None):
        p, P = self.p, self.p.P
        xin = x.unsqueeze(0) if self.scheme == "allgather" else x.view(P, self.T // P, p.H)
        hq_quantize_pack(xin, p.keep_idx, p.rest_idx, self.inv, self.zero, self.codes, self.side, stream=stream)
        return self.codes, self.side

    def exchange(self, codes: torch.Tensor, side: torch.Tensor):
        if self.scheme == "allgather":
            return allgather_stack(codes, self.group), allgather_stack(side, self.group)
        return alltoall_blocks(codes, self.group), alltoall_blocks(side, self.group)

    def reduce_block(self, codes_recv: torch.Tensor, side_recv: torch.Tensor, out: torch.Tensor | None = None,
                     stream=None) -> torch.Tensor:
        """The rank-ordered reduction of the received wire [P, rows, W] / [P, k, rows] into
        [rows, H] bf16: all T rows (allgather) or this rank's row block (reduce_scatter)."""
        p = self.p
        rows = codes_recv.shape[1]
        if out is None:
            out = torch.empty((rows, p.H), dtype=torch.bfloat16, device=codes_recv.device)
        hq_dequant_reduce(codes_recv, side_recv, p.keep_idx, p.rest_idx, p.scale, p.zero, out, stream=stream)
        return out

    def reduce(self, codes_recv: torch.Tensor, side_recv: torch.Tensor, out: torch.Tensor | None = None,
               stream=None) -> torch.Tensor:
        """reduce_block, then for reduce_scatter the reduced row blocks all-gathered into [T, H]."""
        if self.scheme == "allgather":
            return self.reduce_block(codes_recv, side_recv, out, stream=stream)
        full = allgather_rows(self.reduce_block(codes_recv, side_recv, stream=stream), self.group)
        if out is not None:
            out.copy_(full)
            return out
        return full

    def __call__(self, x: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
        codes, side = self.pack(x)
        return self.reduce(*self.exchange(codes, side), out=out)


class PeerAllReduce:
    """Scheme ``peer``: the wires stay where they are written and every rank's reduction reads the
    others' in place.

    ``wires`` is a list of P (codes [T, W] int32, side [k, T] bf16) pairs, entry r rank r's wire as
    this process sees it: for real ranks, the ranks' parts of one symmetric-memory allocation
    (``symmetric_wires``), so that entry r != rank is a peer GPU's memory reached over
    NVLink/NVSwitch.  ``barrier`` orders the ranks: every rank's pack before any reduction, and
    every reduction before the next pack overwrites a wire.  Nothing is gathered: the only data
    movement is the reduction kernel's own loads of the P wires."""

    def __init__(self, params: HybridParams, T: int, rank: int, wires, barrier=None):
        self.p, self.T, self.rank = params, T, rank
        if len(wires) != params.P:
            raise ValueError("one (codes, side) pair per rank")
        _check_row_aligned(params.H)
        self.wires = wires
        self.barrier = barrier or (lambda: None)
        self.inv, self.zero = params.row(rank)

    def pack(self, x: torch.Tensor, stream=None) -> None:
        p = self.p
        codes, side = self.wires[self.rank]
        hq_quantize_pack(x.unsqueeze(0), p.keep_idx, p.rest_idx, self.inv, self.zero, codes.unsqueeze(0),
                         side.unsqueeze(0), stream=stream)

    def reduce(self, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        p = self.p
        if out is None:
            out = torch.empty((self.T, p.H), dtype=torch.bfloat16, device=p.scale.device)
        hq_dequant_reduce_ranks([c for c, _ in self.wires], [s for _, s in self.wires], p.keep_idx, p.rest_idx,
                                p.scale, p.zero, out, stream=stream)
        return out

    def __call__(self, x: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
        self.pack(x)
        self.barrier()   # every rank's wire is written
        out = self.reduce(out)
        self.barrier()   # every rank has read the wires
        return out


def symmetric_wires(params: HybridParams, T: int, group=None, timeout_ms: int = 10000):
    """The P ranks' wire buffers in one symmetric-memory allocation across the group (one process
    per GPU, peer access between the GPUs): returns (wires, barrier) for ``PeerAllReduce``.  The
    barrier is torch's device-side one, bounded by timeout_ms."""
    import torch.distributed._symmetric_memory as symm_mem

    P, H, k = params.P, params.H, params.k
    W = (H - k) // 8
    code_bytes = (T * W * 4 + 255) // 256 * 256
    side_bytes = (k * T * 2 + 255) // 256 * 256
    buf = symm_mem.empty(code_bytes + side_bytes, dtype=torch.uint8, device=params.scale.device)
    hdl = symm_mem.rendezvous(buf, group if group is not None else dist.group.WORLD)
    wires = [(hdl.get_buffer(r, (T, W), torch.int32, 0), hdl.get_buffer(r, (k, T), torch.bfloat16, code_bytes // 2))
             for r in range(P)]
    return wires, (lambda: hdl.barrier(channel=0, timeout_ms=timeout_ms))


# ---------------------------------------------------------------------------------------------
# Two-step: quantized reduce-scatter, then re-quantized all-gather
# ---------------------------------------------------------------------------------------------
@dataclass
class StepTwoParams:
    """Step-2 grids: reducer j quantizes its reduced row block with row j of scale/inv_scale/zero
    [P, H]; the kept set (keep_idx, rest_idx) is shared by all reducers, selected by the same rule
    as step 1 (ranges aggregated over the reducers)."""

    keep_idx: torch.Tensor
    rest_idx: torch.Tensor
    scale: torch.Tensor
    inv_scale: torch.Tensor
    zero: torch.Tensor

    @property
    def k(self) -> int:
        return self.keep_idx.shape[0]


class TwoStepAllReduce:
    """Step 1 is ``HybridAllReduce(scheme="reduce_scatter")`` without its bf16 all-gather; step 2:
    this rank (reducer j) quantizes its reduced block [T/P, H] with its step-2 grid (P = 1), the
    step-2 wires are all-gathered, and every block is dequantized with its reducer's grid
    (P = 1 per block: nothing is summed in step 2)."""

    def __init__(self, params: HybridParams, params2: StepTwoParams, T: int, rank: int, group=None):
        self.step1 = HybridAllReduce(params, T, rank, "reduce_scatter", group)
        self.p2, self.rank, self.group = params2, rank, group
        P, H = params.P, params.H
        self.Tb = T // P
        dev = params.scale.device
        k2 = params2.k
        self.codes2 = torch.empty((1, self.Tb, (H - k2) // 8), dtype=torch.int32, device=dev)
        self.side2 = torch.empty((1, k2, self.Tb), dtype=torch.bfloat16, device=dev)

    # the phases, each a local step between two collectives
    def step1_reduce(self, codes_recv: torch.Tensor, side_recv: torch.Tensor, stream=None) -> torch.Tensor:
        """Step 1's reduction of this reducer's row block (received from every rank), [T/P, H] bf16."""
        return self.step1.reduce_block(codes_recv, side_recv, stream=stream)

    def step2_pack(self, red: torch.Tensor, stream=None):
        """This reducer's block quantized again with its own step-2 grid (P = 1)."""
        p2, j = self.p2, self.rank
        hq_quantize_pack(red.unsqueeze(0), p2.keep_idx, p2.rest_idx, p2.inv_scale[j:j + 1], p2.zero[j:j + 1],
                         self.codes2, self.side2, stream=stream)
        return self.codes2, self.side2

    def step2_unpack(self, codes_all: torch.Tensor, side_all: torch.Tensor, out: torch.Tensor | None = None,
                     stream=None) -> torch.Tensor:
        """Every reducer's step-2 wire [P, T/P, W2] / [P, k2, T/P] dequantized with that reducer's grid
        into its rows of out [T, H] (P = 1 per block: nothing is summed)."""
        p2 = self.p2
        P, H = p2.scale.shape
        if out is None:
            out = torch.empty((P * self.Tb, H), dtype=torch.bfloat16, device=codes_all.device)
        for b in range(P):
            hq_dequant_reduce(codes_all[b:b + 1], side_all[b:b + 1], p2.keep_idx, p2.rest_idx, p2.scale[b:b + 1],
                              p2.zero[b:b + 1], out[b * self.Tb:(b + 1) * self.Tb], stream=stream)
        return out

    def __call__(self, x: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        s1 = self.step1
        red = self.step1_reduce(*s1.exchange(*s1.pack(x, stream=stream)), stream=stream)
        codes2, side2 = self.step2_pack(red, stream=stream)
        return self.step2_unpack(allgather_stack(codes2, self.group), allgather_stack(side2, self.group), out,
                                 stream=stream)


# ---------------------------------------------------------------------------------------------
# The same schemes with the P ranks simulated on one GPU (no collectives)
# ---------------------------------------------------------------------------------------------
def two_step_simulated(x: torch.Tensor, params: HybridParams, params2: StepTwoParams, out1: torch.Tensor,
                       out: torch.Tensor, codes: torch.Tensor, side: torch.Tensor, codes2: torch.Tensor,
                       side2: torch.Tensor, stream=None) -> None:
    """The two-step all-reduce of P simulated ranks x [P, T, H] on one GPU, block by block.

    Step 1 (quantized reduce-scatter): every rank's wire (codes [P, T, W], side [P, k, T]), then
    the rank-ordered reduction of all rows into out1 [T, H] -- the P reducers' blocks side by side.
    Step 2 (re-quantized all-gather): reducer j quantizes rows [j*T/P, (j+1)*T/P) of out1 with its
    own grid into codes2[j] [T/P, W2] and side2[j] [k2, T/P], and each block is dequantized with
    that grid into the same rows of out.  Buffers are the caller's."""
    P, T, H = x.shape
    Tb = T // P
    hq_quantize_pack(x, params.keep_idx, params.rest_idx, params.inv_scale, params.zero, codes, side, stream=stream)
    hq_dequant_reduce(codes, side, params.keep_idx, params.rest_idx, params.scale, params.zero, out1, stream=stream)
    for j in range(P):
        rows = slice(j * Tb, (j + 1) * Tb)
        hq_quantize_pack(out1[rows].unsqueeze(0), params2.keep_idx, params2.rest_idx, params2.inv_scale[j:j + 1],
                         params2.zero[j:j + 1], codes2[j:j + 1], side2[j:j + 1], stream=stream)
        hq_dequant_reduce(codes2[j:j + 1], side2[j:j + 1], params2.keep_idx, params2.rest_idx, params2.scale[j:j + 1],
                          params2.zero[j:j + 1], out[rows], stream=stream)


def step_two_params_simulated(cal_batches, params: HybridParams, k2: int, beta: float) -> StepTwoParams:
    """Step-2 grids from calibration batches [P, T, H] of P simulated ranks: each batch goes
    through step 1, reducer j's moving averages follow its reduced row block (P = 1 calls), and
    the step-2 selection runs over the reducers' statistics [P, H]."""
    P, H = params.P, params.H
    dev = params.scale.device
    emin = torch.empty((P, H), dtype=torch.float32, device=dev)
    emax = torch.empty((P, H), dtype=torch.float32, device=dev)
    for b, xb in enumerate(cal_batches):
        _, T, _ = xb.shape
        Tb = T // P
        k = params.k
        codes = torch.empty((P, T, (H - k) // 8), dtype=torch.int32, device=dev)
        side = torch.empty((P, k, T), dtype=torch.bfloat16, device=dev)
        red = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
        hq_quantize_pack(xb, params.keep_idx, params.rest_idx, params.inv_scale, params.zero, codes, side)
        hq_dequant_reduce(codes, side, params.keep_idx, params.rest_idx, params.scale, params.zero, red)
        for j in range(P):
            hq_calibrate(red[j * Tb:(j + 1) * Tb].unsqueeze(0), emin[j:j + 1], emax[j:j + 1], beta, b == 0)
    p2 = StepTwoParams(keep_idx=torch.empty(k2, dtype=torch.int32, device=dev),
                       rest_idx=torch.empty(H - k2, dtype=torch.int32, device=dev),
                       scale=torch.empty((P, H), dtype=torch.float32, device=dev),
                       inv_scale=torch.empty((P, H), dtype=torch.float32, device=dev),
                       zero=torch.empty((P, H), dtype=torch.uint8, device=dev))
    hq_select_topk(emin, emax, k2, p2.keep_idx, p2.rest_idx, p2.scale, p2.inv_scale, p2.zero)
    return p2

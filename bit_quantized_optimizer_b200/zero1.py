"""ZeRO-1 sharding of the fused 4-bit AdamW step over data-parallel ranks.

Every rank keeps the full fp32 weights and bf16 gradients, each in one flat
buffer, and the optimizer state of its own shard only.  One step is

    reduce-scatter of the gradients (bf16, sum)
      -> the step kernel on the rank's shard (one adamw4 handle per chunk)
      -> all-gather of the updated weights (fp32),

cut into chunks so that the collectives of one chunk overlap the step of
another.  Shards are block-aligned pieces of the tensors; every block's scale
and every random draw are keyed by the element's index in its whole tensor
(``adamw4_tensor.elem_offset``), so the sharded step gives the same bits as the
single-device step on the reduced gradient.

The pages describe the optimizer on one device; the sharding, the flat layout
and the checkpoint merge are this library's.  Collectives go through
``torch.distributed`` (NCCL on GPUs); every step of the method itself runs in
the CUDA kernel behind ``AdamW4``.
"""
from __future__ import annotations

import struct
from dataclasses import dataclass

import numpy as np

from . import (ADAMW4_T_QUANT_STATE, BLOCK, AdamW4, is_fp32_state)

_MAGIC = b"ADAMW4S1"
_HEAD = "<IIqQQ"          # n_tensors, vcode, t, seed, payload_bytes (after the magic)
_REC = "<IIq"             # tensor_id, kind, numel


def _round_up(x: int, m: int) -> int:
    return (x + m - 1) // m * m


@dataclass(frozen=True)
class Piece:
    """The part of tensor ``tensor`` that one rank owns in one chunk."""
    tensor: int         # index in the tensor list
    elem_offset: int    # its first element within the tensor (a multiple of 128)
    numel: int
    flat: int           # index of that element in the flat buffer


class FlatLayout:
    """Tensors placed one after another in a flat buffer, each starting at a
    multiple of 128 elements, then cut into ``chunks`` equal chunks, each cut
    into ``world`` equal shards of ``shard`` elements (a multiple of 128).

    Rank r owns elements [k W S + r S, k W S + (r+1) S) of chunk k.  Every cut
    falls on a block boundary of every tensor, so the pieces are whole blocks
    except for a tensor's own ragged last block.  Shards are equal in elements
    (the collectives need equal parts), not in state bytes: fp32-state tensors
    are small next to the 4-bit ones."""

    def __init__(self, numels, world: int, chunks: int = 1):
        if world < 1 or chunks < 1:
            raise ValueError("world and chunks must be >= 1")
        self.numels = [int(n) for n in numels]
        if any(n <= 0 for n in self.numels):
            raise ValueError("every tensor needs numel > 0")
        self.world, self.chunks = int(world), int(chunks)
        self.offsets = []
        end = 0
        for n in self.numels:
            self.offsets.append(end)
            end = _round_up(end + n, BLOCK)
        self.used = end
        parts = self.world * self.chunks
        self.shard = max(BLOCK, _round_up(-(-end // parts), BLOCK))
        self.padded = self.shard * parts

    def tensor_view(self, flat, i: int):
        """Tensor i as a slice of a flat buffer."""
        return flat[self.offsets[i]:self.offsets[i] + self.numels[i]]

    def chunk_range(self, k: int):
        span = self.world * self.shard
        return k * span, (k + 1) * span

    def shard_range(self, rank: int, k: int):
        lo = self.chunk_range(k)[0] + rank * self.shard
        return lo, lo + self.shard

    def pieces(self, rank: int, k: int):
        """The pieces of rank ``rank`` in chunk ``k``, in tensor order."""
        lo, hi = self.shard_range(rank, k)
        out = []
        for i, (off, n) in enumerate(zip(self.offsets, self.numels)):
            a, b = max(lo, off), min(hi, off + n)
            if a < b:
                out.append(Piece(i, a - off, b - a, a))
        return out


def piece_spec(spec: dict, piece: Piece) -> dict:
    """The descriptor of one piece: the tensor's id, flags and weight decay,
    its elem_offset, and QUANT_STATE when the whole tensor keeps 4-bit state
    (a small piece would otherwise be classified fp32)."""
    flags = int(spec.get("flags", 0))
    if not is_fp32_state(spec["numel"], flags):
        flags |= ADAMW4_T_QUANT_STATE
    return dict(numel=piece.numel, tensor_id=int(spec["tensor_id"]), flags=flags,
                weight_decay=float(spec.get("weight_decay", 0.0)),
                elem_offset=piece.elem_offset)


# ----------------------------------------------------------------------------
# Checkpoints: the pieces' blobs merged into, and cut out of, the blob that one
# handle over the whole tensor list exports (format in include/adamw4.h).
# ----------------------------------------------------------------------------

def _parse(blob: bytes):
    if blob[:8] != _MAGIC:
        raise ValueError("not an adamw4 state blob")
    n, vcode, t, seed, plen = struct.unpack_from(_HEAD, blob, 8)
    if len(blob) != 40 + plen:
        raise ValueError("state blob has the wrong length")
    off, recs = 40, []
    for _ in range(n):
        tid, kind, numel = struct.unpack_from(_REC, blob, off)
        off += 16
        if kind == 0:
            nb = -(-numel // BLOCK)
            sizes = [("mcodes", nb * 64, np.uint8), ("vcodes", nb * 64, np.uint8),
                     ("mscale", nb, np.float32), ("vscale", nb, np.float32)]
        else:
            sizes = [("m", numel, np.float32), ("v", numel, np.float32)]
        rec = dict(tensor_id=tid, kind=kind, numel=numel)
        for name, count, dt in sizes:
            rec[name] = np.frombuffer(blob, dt, count, off)
            off += count * np.dtype(dt).itemsize
        recs.append(rec)
    if off != len(blob):
        raise ValueError("state blob has trailing bytes")
    return dict(vcode=vcode, t=t, seed=seed), recs


def _pack(head: dict, recs) -> bytes:
    parts = []
    for r in recs:
        parts.append(struct.pack(_REC, r["tensor_id"], r["kind"], r["numel"]))
        keys = ("mcodes", "vcodes", "mscale", "vscale") if r["kind"] == 0 else ("m", "v")
        parts += [np.ascontiguousarray(r[k]).tobytes() for k in keys]
    payload = b"".join(parts)
    return _MAGIC + struct.pack(_HEAD, len(recs), head["vcode"], head["t"], head["seed"],
                                len(payload)) + payload


def merge_state(layout: FlatLayout, specs, blobs) -> bytes:
    """One blob for the whole tensor list from ``blobs[(rank, chunk)]`` (the
    blob of that rank's handle for that chunk; absent where it owns nothing)."""
    head, pieces = None, [[] for _ in specs]
    for (rank, k), blob in blobs.items():
        h, recs = _parse(blob)
        if head is None:
            head = h
        elif h != head:
            raise ValueError("state blobs disagree on vcode, step or seed")
        ps = layout.pieces(rank, k)
        if len(ps) != len(recs):
            raise ValueError(f"blob of rank {rank}, chunk {k} does not match the layout")
        for pc, r in zip(ps, recs):
            if r["tensor_id"] != specs[pc.tensor]["tensor_id"] or r["numel"] != pc.numel:
                raise ValueError(f"blob of rank {rank}, chunk {k} does not match the layout")
            pieces[pc.tensor].append((pc.elem_offset, r))
    if head is None:
        raise ValueError("no state blobs")
    out = []
    for i, spec in enumerate(specs):
        got = sorted(pieces[i], key=lambda x: x[0])
        covered = 0
        for e0, r in got:
            if e0 != covered:
                raise ValueError(f"tensor {spec['tensor_id']}: pieces missing or repeated")
            covered += r["numel"]
        if covered != spec["numel"]:
            raise ValueError(f"tensor {spec['tensor_id']}: pieces missing")
        kind = 1 if is_fp32_state(spec["numel"], int(spec.get("flags", 0))) else 0
        if any(r["kind"] != kind for _, r in got):
            raise ValueError(f"tensor {spec['tensor_id']}: piece kind differs from the tensor's")
        keys = ("mcodes", "vcodes", "mscale", "vscale") if kind == 0 else ("m", "v")
        rec = dict(tensor_id=int(spec["tensor_id"]), kind=kind, numel=spec["numel"])
        for key in keys:
            rec[key] = np.concatenate([r[key] for _, r in got])
        out.append(rec)
    return _pack(head, out)


def split_state(layout: FlatLayout, specs, blob: bytes, rank: int, k: int) -> bytes:
    """The blob of the handle of (rank, chunk k), cut out of a whole-list blob."""
    head, recs = _parse(blob)
    if len(recs) != len(specs):
        raise ValueError("blob does not match the tensor list")
    out = []
    for pc in layout.pieces(rank, k):
        r, spec = recs[pc.tensor], specs[pc.tensor]
        if r["tensor_id"] != spec["tensor_id"] or r["numel"] != spec["numel"]:
            raise ValueError("blob does not match the tensor list")
        rec = dict(tensor_id=r["tensor_id"], kind=r["kind"], numel=pc.numel)
        if r["kind"] == 0:
            b0, nb = pc.elem_offset // BLOCK, -(-pc.numel // BLOCK)
            rec["mcodes"] = r["mcodes"][b0 * 64:(b0 + nb) * 64]
            rec["vcodes"] = r["vcodes"][b0 * 64:(b0 + nb) * 64]
            rec["mscale"] = r["mscale"][b0:b0 + nb]
            rec["vscale"] = r["vscale"][b0:b0 + nb]
        else:
            rec["m"] = r["m"][pc.elem_offset:pc.elem_offset + pc.numel]
            rec["v"] = r["v"][pc.elem_offset:pc.elem_offset + pc.numel]
        out.append(rec)
    return _pack(head, out)


# ----------------------------------------------------------------------------
# The sharded optimizer
# ----------------------------------------------------------------------------

class ZeroAdamW4:
    """ZeRO-1 AdamW4 over a process group.

    ``flat_params`` (fp32, or bf16 for bf16 weights -- the all-gather then
    moves half the bytes) and ``flat_grads`` (bf16) are this rank's flat
    buffers of ``layout.padded`` elements; the model's tensors are views
    ``layout.tensor_view(flat, i)``.  ``specs`` lists, per tensor, numel,
    tensor_id, flags and weight_decay.  Gradients are summed over the ranks
    (divide the loss by the world size for a mean).  Padding elements take
    part in the collectives but in no step.

    ``make_stepper(params, grads, specs)`` builds the per-chunk optimizer over
    the rank's pieces; the default is ``AdamW4`` with the given settings."""

    def __init__(self, flat_params, flat_grads, layout: FlatLayout, specs, *, group=None,
                 lr=1e-3, betas=(0.9, 0.999), eps=1e-8, vcode=0, seed=0, total_steps=0,
                 make_stepper=None):
        import torch
        import torch.distributed as dist
        self.group = group
        self.rank = dist.get_rank(group)
        if dist.get_world_size(group) != layout.world:
            raise ValueError("layout.world differs from the process group's size")
        if flat_params.numel() != layout.padded or flat_grads.numel() != layout.padded:
            raise ValueError("flat buffers must hold layout.padded elements")
        if (flat_params.dtype not in (torch.float32, torch.bfloat16)
                or flat_grads.dtype != torch.bfloat16):
            raise TypeError("flat params must be float32 or bfloat16, flat grads bfloat16")
        if len(specs) != len(layout.numels) or any(
                int(s["numel"]) != n for s, n in zip(specs, layout.numels)):
            raise ValueError("specs do not match the layout")
        self.layout, self.specs, self.lr = layout, [dict(s) for s in specs], lr
        if make_stepper is None:
            def make_stepper(params, grads, pspecs):
                return AdamW4(params, grads, pspecs, lr=lr, betas=betas, eps=eps, vcode=vcode,
                              seed=seed, total_steps=total_steps)
        S = layout.shard
        self.grad_shard = torch.zeros(layout.chunks * S, dtype=flat_grads.dtype,
                                      device=flat_grads.device)
        self._gchunk, self._gshard, self._pchunk, self._pshard = [], [], [], []
        self.kernel_events = None   # a list to collect (start, end) events of each step launch
        self.steppers = []
        for k in range(layout.chunks):
            c0, c1 = layout.chunk_range(k)
            s0, s1 = layout.shard_range(self.rank, k)
            self._gchunk.append(flat_grads[c0:c1])
            self._gshard.append(self.grad_shard[k * S:(k + 1) * S])
            self._pchunk.append(flat_params[c0:c1])
            self._pshard.append(flat_params[s0:s1])
            params, grads, pspecs = [], [], []
            for pc in layout.pieces(self.rank, k):
                params.append(flat_params[pc.flat:pc.flat + pc.numel])
                g0 = k * S + pc.flat - s0
                grads.append(self.grad_shard[g0:g0 + pc.numel])
                pspecs.append(piece_spec(self.specs[pc.tensor], pc))
            self.steppers.append(make_stepper(params, grads, pspecs) if params else None)
        self.t = 0

    def step(self, lr=None):
        """Reduce-scatter, step, all-gather.  All reduce-scatters are issued
        first; chunk k's step waits only for its own, and its all-gather is
        issued right after it, so the transfers of other chunks run under it."""
        import torch.distributed as dist
        rs = [dist.reduce_scatter_tensor(self._gshard[k], self._gchunk[k], group=self.group,
                                         async_op=True) for k in range(self.layout.chunks)]
        ag = []
        for k, stepper in enumerate(self.steppers):
            rs[k].wait()
            if stepper is not None:
                if self.kernel_events is not None:      # timing hook (CUDA events)
                    import torch
                    e0, e1 = (torch.cuda.Event(enable_timing=True),
                              torch.cuda.Event(enable_timing=True))
                    e0.record()
                    stepper.step(self.lr if lr is None else lr)
                    e1.record()
                    self.kernel_events.append((e0, e1))
                else:
                    stepper.step(self.lr if lr is None else lr)
            ag.append(dist.all_gather_into_tensor(self._pchunk[k], self._pshard[k],
                                                  group=self.group, async_op=True))
        for w in ag:
            w.wait()
        self.t += 1

    def local_state_blobs(self) -> dict:
        """{(rank, chunk): blob} of this rank's handles."""
        return {(self.rank, k): s.state_dict_blob() for k, s in enumerate(self.steppers)
                if s is not None}

    def consolidated_state(self) -> bytes:
        """The whole-list blob on every rank (the one a single handle over all
        tensors would export); a collective: every rank calls it."""
        import torch.distributed as dist
        parts = [None] * self.layout.world
        dist.all_gather_object(parts, self.local_state_blobs(), group=self.group)
        blobs = {}
        for p in parts:
            blobs.update(p)
        return merge_state(self.layout, self.specs, blobs)

    def close(self):
        """Frees this rank's handles (also done when they are collected)."""
        for s in self.steppers:
            if s is not None and hasattr(s, "close"):
                s.close()
        self.steppers = [None] * len(self.steppers)

    def load_consolidated_state(self, blob: bytes):
        """Loads this rank's pieces from a whole-list blob (saved at any world
        size or chunk count) and takes its step counter."""
        for k, s in enumerate(self.steppers):
            if s is not None:
                s.load_state_blob(split_state(self.layout, self.specs, blob, self.rank, k))
        self.t = _parse(blob)[0]["t"]

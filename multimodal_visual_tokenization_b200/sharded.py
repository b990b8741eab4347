"""Codebook-sharded greedy RVQ encode: the codebook axis split over the ranks of a process group.

For codebook sets larger than one GPU holds.  Rank w keeps codewords [k0_w, k0_w + K_w) of every
level (contiguous, in rank order) and every rank sees all feature rows.  Per level:

  1. each rank finds its shard's nearest codeword of every row with the exact distance
     (``rvq_shard_select``: distance GEMM on the shard, certificate, exact rescan);
  2. the ranks all-gather those (distance, id) pairs, N x 16 bytes per rank (NCCL; a gloo group
     goes through host memory);
  3. every rank applies the overall nearest (lowest distance, then lowest id) to its copy of the
     residual (``rvq_shard_apply``), reading the winning codeword straight from the owner's
     memory through a CUDA IPC mapping (a peer load over NVLink on another GPU).

The quantizer is the pages' greedy residual quantizer (LongCat-2.5 technical blog, "Discrete
Native Resolution Vision Transformer"); the ids equal those of ``Tokenizer.encode`` on the whole
codebook set, because the nearest codeword overall is the nearest among the shards' nearest.

``ShardedTokenizer.local(codebooks, world)`` runs the same kernels for `world` shards held by one
process on one device (the exchange is then a no-op: every shard writes its own block of the
gathered array), which is how the split is checked without several GPUs.
"""
from __future__ import annotations

from . import (RVQ_BF16, RVQ_F32, RVQ_LEVEL_STATS, RVQ_MAX_SHARDS, RVQError, _check, _dtype_code,
               rvq_build_norms, rvq_ipc_close, rvq_ipc_export, rvq_ipc_import, rvq_shard_apply,
               rvq_shard_select, rvq_shard_workspace_size)


def split_codebook(K: int, world: int, unit: int = 256) -> list[int]:
    """Shard sizes for K codewords over `world` ranks, in whole tiles of `unit` codewords where
    there are enough (the distance GEMM's codeword tile), as even as possible, larger shards on
    lower ranks; the last shard takes the ragged tail.  Every shard holds at least one codeword."""
    if world < 1 or K < world:
        raise ValueError("need 1 <= world <= K")
    tiles = -(-K // unit)
    if tiles >= world:
        per = [tiles // world + (1 if r < tiles % world else 0) for r in range(world)]
        sizes = [p * unit for p in per]
        sizes[-1] -= tiles * unit - K
        if sizes[-1] >= 1:
            return sizes
    return [K // world + (1 if r < K % world else 0) for r in range(world)]


def shard_offsets(sizes) -> list[int]:
    """First global codeword id of every shard (prefix sums of the sizes)."""
    out, k = [], 0
    for s in sizes:
        out.append(k)
        k += int(s)
    return out


class _Shard:
    """One shard resident on this process's device, with its rvq_build_norms outputs."""

    def __init__(self, rank, codebooks, k0):
        import torch
        self.rank = rank
        self.codebooks = codebooks.contiguous()
        self.L, self.K, self.D = (int(v) for v in self.codebooks.shape)
        self.k0 = int(k0)
        self.cb_dtype = _dtype_code(self.codebooks)
        dev = self.codebooks.device
        self.norms = torch.empty((self.L, self.K), dtype=torch.float32, device=dev)
        self.stats = torch.empty((self.L, RVQ_LEVEL_STATS), dtype=torch.float32, device=dev)
        self.operand = (torch.empty_like(self.codebooks, dtype=torch.bfloat16)
                        if self.cb_dtype == RVQ_F32 else None)
        _check(rvq_build_norms(self.codebooks, self.cb_dtype, self.L, self.K, self.D, self.norms, self.stats,
                               self.operand), "rvq_build_norms (shard)")


class ShardedTokenizer:
    """Greedy RVQ with the codebook axis split over W ranks.  Use ``from_group`` (one process per
    GPU, this rank's shard) or ``local`` (all shards in this process)."""

    def __init__(self, shards, sizes, peer_ptrs, rank, group=None, imported=()):
        self.shards = shards            # the shards this process holds
        self.sizes = [int(s) for s in sizes]
        self.W = len(self.sizes)
        if not 1 <= self.W <= RVQ_MAX_SHARDS:
            raise ValueError(f"1 <= world <= {RVQ_MAX_SHARDS} shards")
        self.k0 = shard_offsets(self.sizes)
        self.K = sum(self.sizes)
        self.peer_ptrs = list(peer_ptrs)  # rank w's stored codebooks, as seen from this process
        self.rank = rank
        self.group = group
        self._imported = list(imported)   # (ptr, offset) mappings to close
        s0 = shards[0]
        self.L, self.D, self.cb_dtype = s0.L, s0.D, s0.cb_dtype
        self.device = s0.codebooks.device
        self._ws = None

    # ------------------------------------------------------------------ construction
    @classmethod
    def local(cls, codebooks, world, sizes=None):
        """All `world` shards of codebooks [L, K, D] in this process, on codebooks' device."""
        K = int(codebooks.shape[1])
        if not 1 <= world <= RVQ_MAX_SHARDS:
            raise ValueError(f"1 <= world <= {RVQ_MAX_SHARDS} shards")
        sizes = list(sizes) if sizes is not None else split_codebook(K, world)
        if len(sizes) != world or sum(sizes) != K or min(sizes) < 1:
            raise ValueError("shard sizes must be >= 1 and sum to K")
        offs = shard_offsets(sizes)
        shards = [_Shard(w, codebooks[:, offs[w]:offs[w] + sizes[w]], offs[w]) for w in range(world)]
        return cls(shards, sizes, [s.codebooks.data_ptr() for s in shards], rank=None)

    @classmethod
    def from_group(cls, shard_codebooks, group=None):
        """This rank's shard [L, K_w, D] (contiguous ids, rank order) on its own GPU.  Collective:
        every rank of `group` calls it.  Shard sizes and IPC handles of the shards are exchanged
        through the group; every rank must keep its shard alive until ``close``."""
        import torch
        import torch.distributed as dist
        rank, world = dist.get_rank(group), dist.get_world_size(group)
        meta = {"K": int(shard_codebooks.shape[1]), "L": int(shard_codebooks.shape[0]),
                "D": int(shard_codebooks.shape[2]), "dtype": str(shard_codebooks.dtype)}
        metas = [None] * world
        dist.all_gather_object(metas, meta, group=group)
        if any((m["L"], m["D"], m["dtype"]) != (meta["L"], meta["D"], meta["dtype"]) for m in metas):
            raise ValueError("every shard needs the same L, D and dtype")
        sizes = [m["K"] for m in metas]
        shard = _Shard(rank, shard_codebooks, shard_offsets(sizes)[rank])
        torch.cuda.synchronize(shard.codebooks.device)  # shard data final before peers map it
        code, handle, offset = rvq_ipc_export(shard.codebooks)
        _check(code, "rvq_ipc_export")
        handles = [None] * world
        dist.all_gather_object(handles, (handle, offset), group=group)
        ptrs, imported = [], []
        for w, (h, off) in enumerate(handles):
            if w == rank:
                ptrs.append(shard.codebooks.data_ptr())
                continue
            code, p = rvq_ipc_import(h, off)
            _check(code, f"rvq_ipc_import (rank {w})")
            ptrs.append(p)
            imported.append((p, off))
        return cls([shard], sizes, ptrs, rank=rank, group=group, imported=imported)

    def close(self):
        """Unmap the peers' shards (collective for ``from_group``: no rank frees its shard while
        another may still read it)."""
        import torch
        torch.cuda.synchronize(self.device)  # no kernel may still read a mapping
        for p, off in self._imported:
            rvq_ipc_close(p, off)
        self._imported = []
        if self.rank is not None:
            import torch.distributed as dist
            dist.barrier(group=self.group)

    # ------------------------------------------------------------------ encode
    def workspace(self, N):
        import torch
        need = 256
        for s in self.shards:
            code, nbytes = rvq_shard_workspace_size(N, self.D, s.K)
            _check(code, "rvq_shard_workspace_size")
            need = max(need, nbytes)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(need, dtype=torch.uint8, device=self.device)
        return self._ws

    def _exchange(self, sel_all):
        """Give every rank all W blocks of sel_all [W, N, 2]."""
        if self.rank is None:
            return  # local: every shard wrote its own block
        import torch
        import torch.distributed as dist
        mine = sel_all[self.rank].clone()
        if dist.get_backend(self.group) == "nccl":
            dist.all_gather_into_tensor(sel_all, mine, group=self.group)
        else:  # gloo: through host memory
            host = [torch.empty(mine.shape, dtype=mine.dtype) for _ in range(self.W)]
            dist.all_gather(host, mine.cpu(), group=self.group)
            for w in range(self.W):
                sel_all[w].copy_(host[w])

    def encode(self, features, residual=False, status=None, check=True):
        """Greedy RVQ of features [N, D] (the same rows on every rank) -> (ids [N, L] int32,
        residual [N, D] fp32 or None, fallbacks [shards here, L] int32: rows per level that
        needed an exact scan of a shard)."""
        import torch
        N, D = (int(v) for v in features.shape)
        if D != self.D:
            raise ValueError("feature width differs from the codebooks")
        dev = self.device
        ids = torch.empty((N, self.L), dtype=torch.int32, device=dev)
        res = torch.empty((N, D), dtype=torch.float32, device=dev) if residual else None
        fb = torch.zeros((len(self.shards), self.L), dtype=torch.int32, device=dev)
        own_status = status is None and check
        if own_status:
            status = torch.zeros(1, dtype=torch.int32, device=dev)
        ws = self.workspace(N)
        sel_all = torch.empty((self.W, N, 2), dtype=torch.float64, device=dev)
        f_dtype = _dtype_code(features)
        for l in range(self.L):
            for i, s in enumerate(self.shards):
                _check(rvq_shard_select(features, f_dtype, N, D, s.codebooks, s.cb_dtype, s.operand, s.norms,
                                        s.stats, self.L, s.K, s.k0, l, res, sel_all[s.rank], fb[i], ws,
                                        ws.numel(), status), "rvq_shard_select")
            self._exchange(sel_all)
            _check(rvq_shard_apply(features, f_dtype, N, D, sel_all, self.W, self.peer_ptrs, self.cb_dtype,
                                   self.sizes, self.L, l, ids, res, ws, ws.numel(), status), "rvq_shard_apply")
        if own_status:
            code = int(status.item())
            if code != 0:
                raise RVQError(code, "sharded encode (device)")
        return ids, res, fb


__all__ = ["ShardedTokenizer", "split_codebook", "shard_offsets", "RVQ_BF16", "RVQ_F32"]

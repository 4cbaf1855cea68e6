"""Row-sharded C = A.B over the ranks of a process group, with C all-gathered.

Output tiles of a GEMM are independent, so the product splits across G GPUs
with no exchange until the end: rank r holds rows [m0_r, m1_r) of A (its
slab) and all of B, computes rows [m0_r, m1_r) of C with the library's
kernel, and an all-gather then gives every rank the whole M x N C.  This is
the distributed step the tile ledger of "GPU 执行模型" (section "Tile
小账本") leaves to a later chapter: the per-GPU tile work is unchanged, and
only C's slabs cross the interconnect.

One process per GPU (torch.distributed, NCCL over NVLink / NVSwitch on a GPU
node; gloo for host-side tests).  Two forms:

* collective: the slab compute is one ``gemm_bf16`` call writing straight
  into this rank's rows of C (no staging copy); the gather is one broadcast
  per rank of that rank's rows, in rank order, so slabs of unequal height
  need no padding.  Every rank issues the same collectives in the same order.
* fused (``peer_c`` given): one ``gemm_bf16_allgather`` kernel computes the
  slab and its epilogue stores every finished chunk into this rank's C and
  into every other rank's C (their buffers mapped into this process, e.g. by
  CUDA IPC or symmetric memory), so the transfer overlaps the math; a barrier
  then tells every rank that all slabs have landed.  No TMA load reads another
  GPU's memory: only the epilogue's stores cross NVLink.
"""
from __future__ import annotations

from typing import Callable, List, Sequence, Tuple

ROW_BLOCK = 128      # slab boundaries fall on whole 128-row tile blocks


def row_partition(M: int, world: int, block: int = ROW_BLOCK) -> List[Tuple[int, int]]:
    """Balanced row slabs [m0, m1) for `world` ranks, boundaries on whole
    `block`-row blocks (so no output tile straddles two ranks); the first
    ranks take one block more when the blocks do not divide evenly, and
    trailing ranks may get empty slabs when M has fewer blocks than ranks."""
    if M < 0 or world < 1 or block < 1:
        raise ValueError(f"bad partition request: M={M}, world={world}, block={block}")
    blocks = -(-M // block)
    base, extra = divmod(blocks, world)
    out, start = [], 0
    for r in range(world):
        nb = base + (1 if r < extra else 0)
        m0 = min(M, start * block)
        m1 = min(M, (start + nb) * block)
        out.append((m0, m1))
        start += nb
    return out


def slab_of(M: int, rank: int, world: int) -> Tuple[int, int]:
    return row_partition(M, world)[rank]


def gather_rows(C, parts: Sequence[Tuple[int, int]], rank: int, group=None) -> None:
    """Every rank's rows [m0_r, m1_r) of C (a 2-D row-major tensor) reach
    every rank: one broadcast per non-empty slab, from its owner, in rank
    order.  Rows of a row-major matrix are contiguous, so each broadcast
    moves that block of C in place.  With NCCL the broadcasts read and write
    device memory directly (ordered after the current stream's work); with
    gloo (host-side process groups) a device C is staged through host
    memory, one slab at a time."""
    import torch
    import torch.distributed as dist
    device_c = C.is_cuda and dist.get_backend(group) != "nccl"
    if device_c:
        torch.cuda.current_stream().synchronize()
    for r, (m0, m1) in enumerate(parts):
        if m1 <= m0:
            continue
        view = C[m0:m1]
        if not view.is_contiguous():
            raise ValueError("C's row slabs must be contiguous (a row-major matrix)")
        src = dist.get_global_rank(group, r) if group is not None else r
        if device_c:
            host = view.cpu()
            dist.broadcast(host, src=src, group=group)
            if r != rank:
                view.copy_(host)
        else:
            dist.broadcast(view, src=src, group=group)


def gemm_bf16_msharded(A_slab, B, C, M: int, N: int, K: int, c_type: int = 0, group=None, stream=None,
                       slab_gemm: Callable | None = None, peer_c: Sequence | None = None) -> Tuple[int, int]:
    """C = A.B with A's rows sharded over the ranks of `group`.

    A_slab  this rank's rows [m0, m1) of A, a (m1 - m0) x K bf16 tensor,
            row-major (leading dimension A_slab.stride(0));
    B       all of B, stored N x K (K-major), bf16;
    C       the whole M x N output on this rank (fp32 or bf16 per c_type,
            row-major, leading dimension C.stride(0)); on return every rank
            holds all of C.
    stream  the CUDA stream of the slab GEMM (None: the current stream); the
            gather is ordered after it.
    peer_c  fused form: the other ranks' C buffers (tensors or device
            pointers mapped into this process, same shape and leading
            dimension as C), in any order.  This rank's slab is written into
            C and into each of them by one kernel; the call then waits at a
            barrier of `group` until every rank's kernel has finished.
    The slab boundaries are row_partition(M, world).  Returns (m0, m1).

    `slab_gemm(A_slab, B, C_rows, m, N, K, lda, ldb, ldc, c_type, stream)`
    computes one slab; by default the library's gemm_bf16 (the CUDA kernel).
    Host-side tests pass a CPU stand-in here; the product never does.
    """
    import torch.distributed as dist
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    parts = row_partition(M, world)
    m0, m1 = parts[rank]
    if A_slab.shape[0] != m1 - m0:
        raise ValueError(f"rank {rank} holds {A_slab.shape[0]} rows of A; its slab is rows [{m0}, {m1})")
    if C.shape[0] != M or C.shape[1] < N:
        raise ValueError("C must be the whole M x N output on every rank")
    if peer_c is not None:
        import torch
        from . import gemm as G
        if len(peer_c) > 7:
            raise ValueError("the fused form reaches at most 7 other ranks per kernel")
        if m1 > m0:
            G.gemm_bf16_allgather(A_slab, B, [C] + list(peer_c), m1 - m0, N, K, A_slab.stride(0), B.stride(0),
                                  C.stride(0), m0, c_type, stream)
        # every rank's kernel must have finished writing before anyone reads C
        cur = torch.cuda.current_stream()
        if stream is not None and stream != cur:
            cur.wait_stream(stream)
        if dist.get_backend(group) != "nccl":
            cur.synchronize()
        dist.barrier(group=group)
        return m0, m1
    if slab_gemm is None:
        from . import gemm as G
        slab_gemm = G.gemm_bf16
    if m1 > m0:
        slab_gemm(A_slab, B, C[m0:m1], m1 - m0, N, K, A_slab.stride(0), B.stride(0), C.stride(0), c_type,
                  stream)
    if C.is_cuda and stream is not None:
        import torch
        cur = torch.cuda.current_stream()
        if stream != cur:
            cur.wait_stream(stream)
    gather_rows(C, parts, rank, group)
    return m0, m1

"""Host-side logic of the row-sharded GEMM (dense_gemm_engineering_bf16_b200.
sharded) on CPU: the row partition, and the slab compute plus all-gather on
two and three gloo ranks.  The slab compute here is a CPU stand-in built on
the oracle (the test's only way to run without a GPU); the product calls
the CUDA kernel.  Every rank must end with all of C, equal to the oracle's
product of the unsharded matrices, bit for bit."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from dense_gemm_engineering_bf16_b200 import sharded, synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("M", [0, 1, 127, 128, 129, 300, 1000, 4096, 4000])
@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_row_partition_tiles_the_rows(M, world):
    parts = sharded.row_partition(M, world)
    assert len(parts) == world
    assert parts[0][0] == 0 and parts[-1][1] == M
    for (a0, a1), (b0, b1) in zip(parts, parts[1:]):
        assert a1 == b0                                   # contiguous, no overlap
    sizes = [m1 - m0 for m0, m1 in parts]
    assert all(s >= 0 for s in sizes) and sum(sizes) == M
    for m0, m1 in parts:
        if m1 > m0:
            assert m0 % sharded.ROW_BLOCK == 0            # no tile straddles two ranks
    blocks = [-(-s // sharded.ROW_BLOCK) for s in sizes]
    assert max(blocks) - min(blocks) <= 1                 # balanced to one block


def test_row_partition_rejects_bad_requests():
    for args in [(-1, 2), (10, 0)]:
        with pytest.raises(ValueError):
            sharded.row_partition(*args)


def _cpu_slab_gemm(A_slab, B, C_rows, m, N, K, lda, ldb, ldc, c_type, stream):
    """CPU stand-in for the kernel: the oracle's product of the slab, rounded
    once to fp32 and written into this rank's rows of C."""
    import oracle
    a_bits = A_slab.view(torch.int16).numpy().view(np.uint16)
    b_bits = B.view(torch.int16).numpy().view(np.uint16)
    c = oracle.round_f32(oracle.gemm_bf16_f64(a_bits, b_bits, K=K))
    C_rows[:, :N] = torch.from_numpy(c)


def _rank_main(rank, world, port, M, N, K, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        a_bits, b_bits = synth.bf16_operands(M, N, K, "normal", workload=130)
        m0, m1 = sharded.slab_of(M, rank, world)
        A_slab = torch.from_numpy(np.ascontiguousarray(a_bits[m0:m1]).view(np.int16)).view(torch.bfloat16)
        B = torch.from_numpy(b_bits.view(np.int16)).view(torch.bfloat16)
        C = torch.full((M, N), float("nan"), dtype=torch.float32)
        got = sharded.gemm_bf16_msharded(A_slab, B, C, M, N, K, group=None, slab_gemm=_cpu_slab_gemm)
        q.put((rank, got, C.numpy().copy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,M", [(2, 300), (3, 700), (2, 100)])
def test_slabs_and_gather_on_gloo_ranks(world, M):
    import oracle
    N, K = 96, 64
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, M, N, K, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    a_bits, b_bits = synth.bf16_operands(M, N, K, "normal", workload=130)
    want = oracle.round_f32(oracle.gemm_bf16_f64(a_bits, b_bits, K=K))
    parts = sharded.row_partition(M, world)
    for rank, slab, C in results:
        assert tuple(slab) == parts[rank]
        assert np.array_equal(C.view(np.uint32), want.view(np.uint32)), f"rank {rank}: C differs"

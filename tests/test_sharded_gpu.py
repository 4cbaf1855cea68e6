"""The row-sharded GEMM through the CUDA kernel, with two ranks as two
processes sharing the one GPU: each rank computes its slab of C with
gemm_bf16 (the kernels of the two ranks never wait on each other), the slabs
are all-gathered over gloo, and every rank's C must match the oracle's
product of the unsharded matrices.  (On a multi-GPU node the same code runs
one process per GPU over NCCL.)"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, M, N, K, dist_name, q):
    import torch
    import torch.distributed as dist

    from dense_gemm_engineering_bf16_b200 import gemm as G
    from dense_gemm_engineering_bf16_b200 import sharded, synth
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        a_bits, b_bits = synth.bf16_operands(M, N, K, dist_name, workload=131)
        m0, m1 = sharded.slab_of(M, rank, world)
        A_slab = torch.from_numpy(np.ascontiguousarray(a_bits[m0:m1]).view(np.int16)).cuda().view(torch.bfloat16)
        B = torch.from_numpy(b_bits.view(np.int16)).cuda().view(torch.bfloat16)
        C = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        sharded.gemm_bf16_msharded(A_slab, B, C, M, N, K)
        G.gemm_check_device_status()
        q.put((rank, C.cpu().numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("dist_name", ["ints", "normal"])
def test_two_ranks_on_one_gpu_gather_the_whole_product(dist_name):
    import oracle
    from dense_gemm_engineering_bf16_b200 import synth
    world, M, N, K = 2, 1000, 768, 512
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, M, N, K, dist_name, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=300) for _ in range(world)]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    a_bits, b_bits = synth.bf16_operands(M, N, K, dist_name, workload=131)
    c_ref, s_abs = oracle.gemm_bf16_f64(a_bits, b_bits, K=K, with_abs=True)
    for rank, C in results:
        got = C.astype(np.float64)
        if dist_name == "ints":
            assert np.array_equal(got, oracle.round_f32(c_ref).astype(np.float64)), f"rank {rank}"
        else:
            assert np.all(np.abs(got - c_ref) <= 1e-3 * s_abs + 1e-6), f"rank {rank}"


def test_fused_form_writes_every_copy_on_one_rank():
    """The fused form's Python path, one rank (gloo): this rank's slab (all of
    C) goes into C and into two more buffers standing in for other ranks' C."""
    import torch
    import torch.distributed as dist

    import oracle
    from dense_gemm_engineering_bf16_b200 import sharded, synth
    import os
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("gloo", rank=0, world_size=1)
    try:
        M, N, K = 700, 520, 512
        a_bits, b_bits = synth.bf16_operands(M, N, K, "ints", workload=132)
        A = torch.from_numpy(a_bits.view(np.int16)).cuda().view(torch.bfloat16)
        B = torch.from_numpy(b_bits.view(np.int16)).cuda().view(torch.bfloat16)
        C = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        peers = [torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda") for _ in range(2)]
        assert sharded.gemm_bf16_msharded(A, B, C, M, N, K, peer_c=peers) == (0, M)
        want = oracle.round_f32(oracle.gemm_bf16_f64(a_bits, b_bits, K=K))
        for t in [C] + peers:
            assert np.array_equal(t.cpu().numpy().view(np.uint32), want.view(np.uint32))
    finally:
        dist.destroy_process_group()

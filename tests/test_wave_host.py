"""Host side of the one-way K/V publication (block_causal_streaming_b200.wave) on the CPU.

Two gloo ranks exchange the (faked) IPC handles of their pools and flag arrays the way
PublishedPools does on GPUs; the data path itself (wf_kv_append_publish, the flag waits) is
covered by tests/test_gpu_publish.py on one GPU.  Argument checks of the new entry points run
without a device."""
import ctypes
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from block_causal_streaming_b200 import wave
from block_causal_streaming_b200 import build as wf_build


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _fake_ipc(rank):
    """Stand-ins for wf_ipc_export/import/close: a handle encodes (owner rank, pointer); an
    imported pointer is marked so the test can tell it from a local one."""
    from block_causal_streaming_b200 import _abi
    closed = []

    def export(ptr):
        return (rank.to_bytes(4, "little") + int(ptr).to_bytes(8, "little")).ljust(64, b"\0"), 0

    def imp(exported):
        handle, off = exported
        owner = int.from_bytes(handle[:4], "little")
        assert owner != rank, "a rank must not import its own handle"
        ptr = int.from_bytes(handle[4:12], "little") & ((1 << 48) - 1)
        return (1 << 60) | (owner << 48) | ptr

    _abi.ipc_export = export
    _abi.ipc_import = imp
    _abi.ipc_close = closed.append
    return closed


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        closed = _fake_ipc(rank)
        k = torch.zeros(1024, dtype=torch.bfloat16)
        v = torch.zeros(1024, dtype=torch.bfloat16)
        flags = wave.new_flags(3, "cpu")
        pools = wave.PublishedPools(k, v, flags)
        own = pools.peer(rank)
        others = {r: pools.peer(r) for r in range(world) if r != rank}
        dests = pools.destinations(wave.consumers_of(rank, world))
        pools.close()
        results[rank] = (own, (k.data_ptr(), v.data_ptr(), flags.data_ptr()), others, dests,
                         sorted(closed))
    finally:
        dist.destroy_process_group()


def test_published_pools_exchange_handles_between_two_ranks():
    world, port = 2, _free_port()
    with mp.get_context("spawn").Manager() as m:
        results = m.dict()
        mp.start_processes(_worker, args=(world, port, results), nprocs=world,
                           start_method="spawn", join=True)
        res = dict(results)
    assert set(res) == {0, 1}
    for rank, (own, local, others, dests, closed) in res.items():
        assert own == local                                   # own allocations, not mapped
        (other_rank, ptrs), = others.items()
        assert other_rank == 1 - rank
        _, other_local, _, _, _ = res[other_rank]
        for p, q_local in zip(ptrs, other_local):             # mapped from the other's handles
            assert p >> 60 == 1 and (p >> 48) & 0xFFF == other_rank
            assert p & ((1 << 48) - 1) == q_local & ((1 << 48) - 1)
        assert sorted(closed) == sorted(ptrs)                 # every mapping closed once
    assert res[0][3] == [res[0][2][1]]                        # rank 0 publishes to rank 1
    assert res[1][3] == []                                    # the last rank to nobody


def test_consumers_follow_the_wavefront():
    assert wave.consumers_of(0, 4) == [1, 2, 3]
    assert wave.consumers_of(2, 4) == [3]
    assert wave.consumers_of(3, 4) == []
    assert tuple(wave.new_flags(5, "cpu").shape) == (5, wave.WF_MAX_CHUNKS)


FAKE = 0x10000


@pytest.fixture(scope="module")
def abi():
    wf_build.build()
    from block_causal_streaming_b200 import _abi
    return _abi


def test_publish_argument_checks_without_a_gpu(abi):
    desc = abi.WavefrontDesc([0, 64, 128, 200], [0, 200, 1000], 1, 8)
    pool = abi.KvPool(k_pool=FAKE, v_pool=FAKE, num_pages=8, page_size=64, num_heads=2,
                      head_dim=128)
    pt = ctypes.cast(ctypes.c_void_p(FAKE), ctypes.POINTER(ctypes.c_int32))
    peers = (abi.PoolDst * 9)(*[abi.PoolDst(FAKE, FAKE, FAKE) for _ in range(9)])

    def publish(n_peers, arr=peers, chunk=1, flags=FAKE):
        return abi.lib.wf_kv_append_publish(ctypes.byref(pool), flags, arr, n_peers, 0, chunk,
                                            FAKE, FAKE, pt, ctypes.byref(desc.c), 3, None)
    assert publish(9) == abi.WF_ERR_INVALID_ARG                    # at most 8 peers
    assert publish(-1) == abi.WF_ERR_INVALID_ARG
    assert publish(1, arr=None) == abi.WF_ERR_INVALID_ARG
    bad = (abi.PoolDst * 1)(abi.PoolDst(FAKE + 8, FAKE, FAKE))
    assert publish(1, arr=bad) == abi.WF_ERR_INVALID_ARG           # misaligned peer pool
    assert publish(1, flags=FAKE + 2) == abi.WF_ERR_INVALID_ARG    # misaligned flags
    assert publish(1, chunk=3) == abi.WF_ERR_INVALID_ARG           # no such chunk

    def published(flags_row, splits=0):
        return abi.lib.wf_attn_forward_published(
            FAKE, ctypes.byref(pool), pt, ctypes.byref(desc.c), 0.1, FAKE, None, flags_row, 1,
            splits, None, 0, None)
    assert published(None) == abi.WF_ERR_INVALID_ARG
    assert published(FAKE + 1) == abi.WF_ERR_INVALID_ARG
    assert published(FAKE, splits=-2) == abi.WF_ERR_INVALID_ARG


def _shared_alloc_worker(rank, world, port, results):
    """Both pools and an FP8 pool exported from one fake allocation per rank: every tensor has
    the same handle and its own offset, so the peer must map the allocation once, derive every
    pointer from that one mapping, and close it once."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from block_causal_streaming_b200 import _abi
        base = 0x7000_0000 + 0x100_0000 * rank
        imports, closed = [], []

        def export(ptr):
            return (rank.to_bytes(4, "little") + base.to_bytes(8, "little")).ljust(64, b"\0"), \
                int(ptr) - base

        def imp(exported):
            handle, off = exported
            imports.append((handle[:4], off))
            return 0x9000_0000 + 0x100_0000 * int.from_bytes(handle[:4], "little") + off

        _abi.ipc_export, _abi.ipc_import, _abi.ipc_close = export, imp, closed.append
        t = [torch.zeros(4, dtype=torch.int32) for _ in range(7)]
        ptrs = {}

        class T:                      # a tensor stand-in at a chosen address inside the block
            def __init__(self, addr):
                self.addr = addr

            def data_ptr(self):
                return self.addr
        own = [T(base + 256 * i) for i in range(7)]
        pools = wave.PublishedPools(own[0], own[1], own[2], fp8=own[3:])
        other = 1 - rank
        results[rank] = (pools.peer(other), pools.peer_fp8(other),
                         pools.destinations_fp8([0, 1]), list(imports))
        pools.close()
        results[rank] = results[rank] + (list(closed),)
        del t, ptrs
    finally:
        dist.destroy_process_group()


def test_tensors_of_one_allocation_are_mapped_once():
    world, port = 2, _free_port()
    with mp.get_context("spawn").Manager() as m:
        results = m.dict()
        mp.start_processes(_shared_alloc_worker, args=(world, port, results), nprocs=world,
                           start_method="spawn", join=True)
        res = dict(results)
    for rank, (peer, peer_fp8, dests, imports, closed) in res.items():
        other = 1 - rank
        mapped = 0x9000_0000 + 0x100_0000 * other
        assert len(imports) == 1 and len(closed) == 1                  # one allocation, once
        assert peer == (mapped, mapped + 256, mapped + 512)
        assert peer_fp8 == (mapped + 768, mapped + 1024, mapped + 1280, mapped + 1536,
                            mapped + 512)                              # flags come last
        assert dests == [peer_fp8]


def _mixed_fp8_worker(rank, world, port, results):
    """Rank 0 passes an FP8 pool, rank 1 none: both ranks see every rank's handles after the one
    exchange, so both refuse the same way and neither waits in a collective for the other."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        _fake_ipc(rank)
        k, v = torch.zeros(64, dtype=torch.bfloat16), torch.zeros(64, dtype=torch.bfloat16)
        flags = wave.new_flags(1, "cpu")
        fp8 = [torch.zeros(64, dtype=torch.uint8) for _ in range(2)] + \
            [torch.zeros(8, dtype=torch.float32) for _ in range(2)]
        try:
            wave.PublishedPools(k, v, flags, fp8=fp8 if rank == 0 else None)
            results[rank] = "accepted"
        except ValueError as e:
            results[rank] = str(e)
        dist.barrier()                      # both ranks still reach the next collective
    finally:
        dist.destroy_process_group()


def test_an_fp8_pool_on_some_ranks_only_is_refused_everywhere():
    world, port = 2, _free_port()
    with mp.get_context("spawn").Manager() as m:
        results = m.dict()
        mp.start_processes(_mixed_fp8_worker, args=(world, port, results), nprocs=world,
                           start_method="spawn", join=True)
        res = dict(results)
    assert set(res) == {0, 1}
    assert all("FP8 pool" in msg for msg in res.values()), res

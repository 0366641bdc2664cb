"""One-way K/V publication between two processes on one GPU, through real CUDA IPC mappings.

Two ranks (processes) stand for two Wave-Parallelism GPUs: rank r owns query chunk
num_ctx + r.  Each maps the other's pools and flag array with wf_ipc_export / wf_ipc_import
(exchanged over a gloo group), publishes its chunk -- bf16 and FP8 -- into its own pools and
the other rank's, and then attends to its own view on its own pool: the bf16 pool through
wf_attn_forward_published, the FP8 pool through wf_kv_dequant_published + wf_attn_forward.
That runs the IPC mapping and the system-scope release / acquire of the flags between two
processes for real.

Both processes share the one device, so their kernels never run concurrently here: the phases
are serialized by host barriers (one rank launches, synchronizes, then the next), and every flag
a kernel waits for is checked on the host before that kernel is launched.  No kernel ever waits
for another process.
"""
import datetime
import os
import socket
import traceback

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

WORLD = 2
GEN = 5
BF16_LAYER, FP8_LAYER = 1, 0      # flag rows: bf16 publication in layer 1, FP8 in layer 0


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _case():
    from block_causal_streaming_b200.workloads import small_case
    # one context chunk, then the chunks of rank 0 and rank 1; 200 and 170 tokens straddle pages
    return small_case("two_process", 2, 128, (130,), (200, 170), 64, seed=71)


def _rank_main(rank, port, results):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(WORLD))
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD,
                            timeout=datetime.timedelta(seconds=120))
    pools = None
    try:
        import oracle
        from oracle import fp8 as ofp8
        import block_causal_streaming_b200 as wf
        from block_causal_streaming_b200 import WavefrontDesc
        from block_causal_streaming_b200.layer import PagedPool, PagedPoolFp8, WavefrontLayer
        from block_causal_streaming_b200.wave import PublishedPools, new_flags
        from block_causal_streaming_b200.workloads import make_inputs

        wl = _case()
        inp = make_inputs(wl)                            # the same seeded data in both ranks
        off, nctx = wl.chunk_offsets, wl.num_ctx_chunks
        own_chunk = nctx + rank
        dev = torch.device("cuda", 0)
        pool = PagedPool(wl.num_pages, wl.page_size, wl.heads, wl.head_dim, dev,
                         fill=float("nan"))
        fp = PagedPoolFp8(wl.num_pages, wl.page_size, wl.heads, wl.head_dim, dev)
        flags = new_flags(2, dev)
        pools = PublishedPools(pool.k, pool.v, flags, fp8=fp.tensors)
        pt = torch.stack([inp.page_table, inp.page_table]).to(dev).contiguous()
        desc = WavefrontDesc(off, wl.chunk_stage, nctx, pt.shape[1])
        k, v = inp.k.to(dev), inp.v.to(dev)
        other = 1 - rank

        # ---- publication, one rank at a time: rank 0 also publishes the context chunk
        for phase in range(WORLD):
            if phase == rank:
                for c in ([0] if rank == 0 else []) + [own_chunk]:
                    wf.kv_append_publish(pool.k, pool.v, flags, pools.destinations([other]),
                                         BF16_LAYER, c, k[off[c]:off[c + 1]],
                                         v[off[c]:off[c + 1]], pt, desc, GEN)
                    wf.kv_append_publish_fp8(*fp.tensors, flags, pools.destinations_fp8([other]),
                                             FP8_LAYER, c, k[off[c]:off[c + 1]],
                                             v[off[c]:off[c + 1]], pt, desc, GEN)
                torch.cuda.synchronize()
                assert wf.check_status() == wf.WF_OK
            dist.barrier()

        # ---- every chunk is now in both ranks' pools: check on the host, before any wait
        f = flags.cpu()
        published = [0, nctx, nctx + 1]
        assert all(int(f[BF16_LAYER, c]) == GEN and int(f[FP8_LAYER, c]) == GEN
                   for c in published), f"flags of rank {rank}: {f[:, :4].tolist()}"
        pt_np = inp.page_table.numpy()
        expect = {}
        for name, src in (("k", inp.k), ("v", inp.v)):
            ref = np.full(tuple(pool.k.shape), 0x7FC0, np.int16)        # bf16 NaN fill
            for c in published:
                oracle.scatter_chunk(ref, pt_np, off[c],
                                     src.view(torch.int16).numpy()[off[c]:off[c + 1]])
            got = (pool.k if name == "k" else pool.v).cpu().view(torch.int16).numpy()
            assert np.array_equal(got, ref), f"rank {rank}: bf16 {name} pool"
            codes, scale = ofp8.quantize_rows(src.float().numpy())
            expect[name] = (codes, scale)
            got_codes = (fp.k_codes if name == "k" else fp.v_codes).cpu().numpy()
            got_codes = oracle.gather_logical(got_codes, pt_np, off[-1])
            assert np.array_equal(got_codes, codes), f"rank {rank}: FP8 {name} codes"

        # ---- attention on this rank's own view, one rank at a time
        view_end = own_chunk + 1
        view = WavefrontDesc(off[:view_end + 1], wl.chunk_stage[:view_end], own_chunk,
                             pt.shape[1])
        q = inp.q[off[own_chunk] - off[nctx]:off[view_end] - off[nctx]].to(dev).contiguous()
        scale = 1.0 / wl.head_dim ** 0.5
        errs = {}
        for phase in range(WORLD):
            if phase == rank:
                out = torch.empty_like(q)
                wf.attn_forward_published(q, pool.k, pool.v, pt[BF16_LAYER], view, scale, out,
                                          flags[BF16_LAYER], GEN, splits=1)
                bf = PagedPool(wl.num_pages, wl.page_size, wl.heads, wl.head_dim, dev,
                               fill=float("nan"))
                for c in range(view_end):
                    wf.kv_dequant_published(*fp.tensors, bf.k, bf.v, FP8_LAYER, c, pt, view,
                                            flags[FP8_LAYER], GEN)
                out8 = torch.empty_like(q)
                WavefrontLayer(bf, pt, FP8_LAYER, off[:view_end + 1], wl.chunk_stage[:view_end],
                               own_chunk).forward(q, out8, scale=scale)
                torch.cuda.synchronize()
                assert wf.check_status() == wf.WF_OK
                n = off[view_end]
                ref = oracle.attention(q.cpu(), inp.k[:n], inp.v[:n], off[:view_end + 1],
                                       own_chunk, scale)
                k8, v8 = (ofp8.dequantize_rows(*(x[0][:n], x[1][:n]))
                          for x in (expect["k"], expect["v"]))
                ref8 = oracle.attention(q.cpu(), k8, v8, off[:view_end + 1], own_chunk, scale)
                for name, got, want in (("bf16", out, ref), ("fp8", out8, ref8)):
                    e = np.abs(got.float().cpu().numpy() - want)
                    errs[name] = (float(e.max()), float(e.mean()))
            dist.barrier()
        results[rank] = ("ok", errs)
    except Exception:
        results[rank] = ("error", traceback.format_exc())
    finally:
        try:
            if pools is not None:
                torch.cuda.synchronize()
                dist.barrier()
                pools.close()
        finally:
            dist.destroy_process_group()


def test_two_processes_publish_into_each_other_and_attend():
    with mp.get_context("spawn").Manager() as m:
        results = m.dict()
        mp.start_processes(_rank_main, args=(_free_port(), results), nprocs=WORLD,
                           start_method="spawn", join=True)
        res = dict(results)
    assert set(res) == {0, 1}, res
    for rank, (status, detail) in res.items():
        assert status == "ok", f"rank {rank}:\n{detail}"
        for name, (mx, mean) in detail.items():
            print(f"rank {rank} {name}: max-abs {mx:.3e}, mean-abs {mean:.3e}")
            assert mx <= 1e-2 and mean <= 1e-3, (rank, name, mx, mean)

"""The peer-memory expert-parallel exchange across processes: two ranks, each
in its own process, on the one GPU this run has, map each other's buffers
through CUDA IPC (moe_ipc_get_handle / moe_ipc_open) and run ep_forward_peer:
the dispatch kernel of each rank stores into the other process's receive
buffer, the down projection of each rank into the other's return buffer.
The phases are ordered on the host (device synchronise, then a gloo barrier);
no kernel waits on the other process.  Each rank's output must equal
moe_forward over the whole batch, bit for bit, on its token shard, for a
bf16 layer and for an E4M3 one (rows exchanged as 1x128 codes with their
scales, outputs returned in bf16)."""
import dataclasses
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, n_redundant, fp8, out):
    sys.path.insert(0, ROOT)
    import datetime

    import numpy as np
    import torch.distributed as dist

    import bench
    import forward_moe_route_b200 as moe
    from forward_moe_route_b200 import ep
    from synth import recipes
    try:
        torch.cuda.set_device(0)
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        dist.init_process_group("gloo", rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=60))
        cfg = dataclasses.replace(
            recipes.small_variant(recipes.CONFIGS["v3_bf16"], T=777, d=512, inter=256,
                                  n_routed=32), n_group=4, topk_group=2,
            dtype="e4m3" if fp8 else "bf16")
        inp = recipes.device_inputs(cfg)
        if fp8:                                  # 128x128 E4M3 expert weights
            E, I, d = cfg.n_experts, cfg.inter, cfg.d
            gq = torch.empty(E, 2 * I, d, dtype=torch.uint8, device="cuda")
            gs = torch.empty(E, 2 * I // 128, d // 128, dtype=torch.float32, device="cuda")
            dq = torch.empty(E, d, I, dtype=torch.uint8, device="cuda")
            ds = torch.empty(E, d // 128, I // 128, dtype=torch.float32, device="cuda")
            moe.moe_quantize_fp8_blockwise(inp["w_gu"], 2 * I, d, E, gq, gs)
            moe.moe_quantize_fp8_blockwise(inp["w_down"], d, I, E, dq, ds)
            inp.update(w_gu=gq, w_gu_scale=gs, w_down=dq, w_down_scale=ds)
        desc_all = moe.desc_from_config(cfg)
        ws_all = moe.workspace(desc_all)
        h_ref = torch.empty(cfg.T, cfg.d, dtype=torch.bfloat16, device="cuda")
        counts = torch.empty(cfg.n_routed, dtype=torch.int32, device="cuda")
        moe.moe_forward(desc_all, inp["x"], None, inp["w_r"], inp["bias"], inp["w_gu"],
                        inp.get("w_gu_scale"), inp["w_down"], inp.get("w_down_scale"), h_ref,
                        None, counts, ws_all)
        replicas = ep.choose_replicas(counts.cpu().numpy(), world, n_redundant) \
            if n_redundant else {}
        pl = ep.Placement(cfg.n_routed, world, replicas)
        lo, hi = bench.token_shard(cfg.T, rank, world)
        c = dataclasses.replace(cfg, T=hi - lo)
        desc = moe.desc_from_config(c)
        x = inp["x"][lo:hi].contiguous()
        full = (inp["w_gu"], inp["w_down"]) + \
            ((inp["w_gu_scale"], inp["w_down_scale"]) if fp8 else ())
        wl = ep.local_weights(pl, rank, cfg.n_shared, *full)
        w_gu, w_down = wl[:2]
        scales = wl[2:] if fp8 else (None, None)
        ex = ep.PeerExchange(desc, pl, rank, cfg.T * cfg.top_k, "cuda", torch.bfloat16)
        ex.open_peers()
        outs = []
        for _ in range(2):                      # twice: the buffers are reused
            h, n = ep.ep_forward_peer(desc, pl, rank, x, None, inp["w_r"], inp["bias"], w_gu,
                                      w_down, ex, w_gu_scale=scales[0], w_down_scale=scales[1])
            torch.cuda.synchronize()
            outs.append((bool(torch.equal(h, h_ref[lo:hi])), int(n)))
        st = moe.moe_last_device_status()
        dist.barrier()
        ex.close()
        dist.destroy_process_group()
        out.put((rank, outs, st, None))
    except Exception as e:  # reported to the parent
        out.put((rank, None, None, repr(e)))


@pytest.mark.parametrize("n_redundant,fp8", [(0, False), (4, False), (4, True)])
def test_ipc_peer_exchange_two_processes(n_redundant, fp8):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, n_redundant, fp8, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = {}
    try:
        for _ in range(2):
            rank, outs, st, err = q.get(timeout=240)
            results[rank] = (outs, st, err)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    for rank in range(2):
        outs, st, err = results[rank]
        assert err is None, f"rank {rank}: {err}"
        assert st == 0, f"rank {rank}: device status {st}"
        assert all(ok for ok, _ in outs), f"rank {rank}: output differs from moe_forward"
        print(f"rank {rank}: rows processed {[n for _, n in outs]}")
    assert sum(results[r][0][0][1] for r in range(2)) == 777 * 8

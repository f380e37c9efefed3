"""Matrix-ownership sharding around the real CUDA step.

Two processes share the one GPU and exchange through gloo (CUDA tensors, no NVLS, no
multicast; the two processes' kernels never wait on each other).  Each rank runs
muon_step_batched on the matrices it owns (longest-processing-time assignment on the
Newton-Schulz FLOPs), keeps only their momentum, and then every weight is broadcast from
its owner.  After two steps every rank's weights must equal, bit for bit, those of a
single-process muon_step_batched over the whole set, and the owners' momentum buffers
those of the single-process run.  Two sampled matrices are held to the oracle: the
orthogonalised update within the bf16 bound, the weight within one storage ulp of the
exact update evaluated with the GPU's own O (prism.simon-ai.net/article/8795, sections on
the ZeRO-like gather of whole matrices and the knapsack assignment of matrices to GPUs).
"""
import datetime
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

SHAPES = [(96, 288), (96, 96), (96, 384), (384, 96), (136, 264), (768, 2304), (3072, 768), (256, 256)]
SAMPLE = (5, 6)          # 768 x 2304 (wide) and 3072 x 768 (tall)
LR, BETA, WD = 0.02, 0.95, 0.1


def _make_set(mb, workloads):
    r = workloads.rng(1301)
    mats = []
    for i, (rows, cols) in enumerate(SHAPES):
        W = torch.tensor(r.standard_normal((rows, cols)) * 0.02, dtype=torch.float32).to(torch.bfloat16).cuda()
        G = torch.tensor(r.standard_normal((rows, cols)) * 1e-3, dtype=torch.float32).to(torch.bfloat16).cuda()
        M = torch.zeros((rows, cols), dtype=torch.float32, device="cuda")
        O = torch.empty((rows, cols), dtype=torch.bfloat16, device="cuda") if i in SAMPLE else None
        mats.append(mb.Matrix(W, G, M, O))
    return mats


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    try:
        import sys
        sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
        import oracle as orc
        from gpu_helpers import assert_update_within_bound, host, rel_f
        from matrix_orthogonalising_optimizer_02_b200 import binding as mb
        from matrix_orthogonalising_optimizer_02_b200 import workloads
        from matrix_orthogonalising_optimizer_02_b200.sharded import ShardedMuonStep

        torch.cuda.set_device(0)
        dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
        hp = mb.hyper(lr=LR, beta=BETA, weight_decay=WD)
        mats = _make_set(mb, workloads)          # identical on every rank (host-seeded draws)
        ref = _make_set(mb, workloads)
        before = {i: (host(mats[i].W), host(mats[i].G)) for i in SAMPLE}
        workspaces = {}

        def step_owned(indices):
            sub = [mats[i] for i in indices]
            key = tuple(indices)
            if key not in workspaces:
                workspaces[key] = mb.workspace(mb.muon_step_workspace_size(sub, hp))
            mb.muon_step_batched(sub, hp, workspaces[key])
            assert mb.device_status(workspaces[key]) == mb.MUON_OK   # synchronises the stream
            torch.cuda.synchronize()

        sharded = ShardedMuonStep([m.W for m in mats], step_owned)
        assert 0 < len(sharded.owned) < len(SHAPES)          # both ranks compute something
        ws_ref = mb.workspace(mb.muon_step_workspace_size(ref, hp))
        for step in range(2):
            sharded.step()
            torch.cuda.synchronize()
            mb.muon_step_batched(ref, hp, ws_ref)
            assert mb.device_status(ws_ref) == mb.MUON_OK
            if step == 0:
                # the oracle on two sampled matrices after the first step (zero momentum: M1 = G)
                for i in SAMPLE:
                    W0, G = before[i]
                    O = host(ref[i].O_out)
                    O_ref = orc.newton_schulz(orc.ns_input(G), orc.fixed_schedule(5))
                    assert rel_f(O, O_ref) <= 2e-2
                    s = orc.scale_factor(*W0.shape, "moonlight")
                    assert_update_within_bound(host(mats[i].W), W0, O, LR, WD, s, bf16=True)
        for i, (m, r) in enumerate(zip(mats, ref)):
            assert torch.equal(m.W, r.W), f"matrix {i}: sharded weights differ from the single-process step"
            if sharded.owner[i] == rank:
                assert torch.equal(m.M, r.M), f"matrix {i}: owner's momentum differs"
        # every rank ends with the same weights
        sums = torch.tensor([float(sum(m.W.double().sum().item() for m in mats))])
        gathered = [torch.zeros(1) for _ in range(world)]
        dist.all_gather(gathered, sums)
        assert all(torch.equal(x, gathered[0]) for x in gathered)
        q.put((rank, "ok"))
    except Exception as e:  # reported to the parent
        import traceback
        q.put((rank, repr(e) + "\n" + traceback.format_exc()))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_sharded_step_with_the_cuda_step_matches_single_process():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = {}
    for _ in procs:
        rank, msg = q.get(timeout=600)
        results[rank] = msg
    for p in procs:
        p.join(timeout=60)
    assert results == {r: "ok" for r in range(world)}, results

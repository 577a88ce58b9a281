"""The FP8 communication layer (fp8_dynamic_scaled_b200.comm) on two gloo ranks on
CPU: the amax all-reduce, per-tensor scaling of a row-sharded tensor and the FP8
all-gather, with the device operations supplied by the oracle so that the
orchestration can run without a GPU.  Expected values: the oracle's quantisation of
the whole (unsharded) tensor."""
import os
import socket
import sys

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

ROWS, COLS = 8, 64          # per rank


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_ops():
    import oracle
    from fp8_dynamic_scaled_b200.comm import DeviceOps

    def bits(x):
        return x.contiguous().view(torch.int16).numpy().view(np.uint16)

    def amax(x):
        return torch.tensor([oracle.amax(bits(x))], dtype=torch.float32)

    def quantize_with_amax(x, fmt, a):
        q, s, _ = oracle.quantize_with_amax(bits(x), fmt, float(a.item()), dequant=False)
        return torch.from_numpy(q), torch.tensor([float(s)], dtype=torch.float32)

    def quantize(x, fmt, mode):
        q, s, _ = oracle.quantize(bits(x), fmt, mode, dequant=False)
        return torch.from_numpy(q), torch.from_numpy(np.ascontiguousarray(s))

    return DeviceOps(amax, quantize_with_amax, quantize)


def _full_tensor(world):
    """The whole tensor; the largest magnitude sits in the last rank's rows."""
    from fp8_dynamic_scaled_b200 import inputs
    g = np.random.default_rng(7)
    x = g.standard_normal((world * ROWS, COLS)).astype(np.float32)
    x[-1, 5] = 300.0
    return inputs.bf16_bits(x)


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from fp8_dynamic_scaled_b200 import comm
        ops = _oracle_ops()
        full = _full_tensor(world)
        mine = full[rank * ROWS:(rank + 1) * ROWS]
        x = torch.from_numpy(mine.view(np.int16)).view(torch.bfloat16)
        res = {}
        res["amax"] = float(comm.global_amax(x, ops=ops).item()) == oracle.amax(full)
        q_ref, s_ref, _ = oracle.quantize(full, oracle.E4M3, oracle.TENSOR, dequant=False)
        q, s = comm.quantize_tensor_sharded(x, oracle.E4M3, ops=ops)
        res["sharded_scale"] = float(s.item()) == float(s_ref[0])
        res["sharded_codes"] = bool(np.array_equal(q.numpy(), q_ref[rank * ROWS:(rank + 1) * ROWS]))
        # without the exchange, rank 0 would pick a different scale for its shard
        q_loc, s_loc, _ = oracle.quantize(mine, oracle.E4M3, oracle.TENSOR, dequant=False)
        res["local_differs"] = rank == world - 1 or float(s_loc[0]) != float(s_ref[0])
        qg, sg = comm.all_gather_fp8(x, oracle.E4M3, comm.FP8_SCALE_TENSOR, ops=ops)
        res["gather_tensor"] = bool(np.array_equal(qg.numpy(), q_ref)) and float(sg.item()) == float(s_ref[0])
        q_row, s_row, _ = oracle.quantize(full, oracle.E5M2, oracle.ROW, dequant=False)
        qg, sg = comm.all_gather_fp8(x, oracle.E5M2, comm.FP8_SCALE_ROW, ops=ops)
        res["gather_row"] = bool(np.array_equal(qg.numpy(), q_row)) and bool(np.array_equal(sg.numpy(), s_row))
        b = comm.payload_bytes(ROWS, COLS, comm.FP8_SCALE_ROW)
        res["bytes"] = b["fp8"] == ROWS * COLS + 4 * ROWS and b["bf16"] == 2 * ROWS * COLS
        out[rank] = res
    finally:
        dist.destroy_process_group()


def test_fp8_comm_two_gloo_ranks():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
        res = dict(out)
    for rank in range(world):
        assert all(res[rank].values()), (rank, res[rank])

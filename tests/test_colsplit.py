"""Column-parallel split (bit_quantized_linear_qmm_b200.colsplit) on CPU: two gloo ranks each take
their block of a layer's outputs, compute it with the oracle, and the all-gathered y must equal the
unsplit layer exactly (each output depends on its own weights and x only).  Covers every weight
format's block layout: rows, int4 columns, per-group scale columns and BitLinear's packed rows."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _layers():
    """(fmt, N, full weights, function(weights) -> y (double [M, N])) for each format (oracle)."""
    import oracle
    import synth
    M, K = 3, 512
    x = synth.activations(90, (M, K), "f32").vals
    out = []
    N = 200
    w = synth.normal(91, (N, K), 0.02)
    codes, s, b = oracle.affine_quantize(w, 4, 64, False)
    bias = synth.normal(92, (N,), 0.01)
    out.append(("affine", N, {"codes": codes, "scales": s, "biases": b, "bias": bias},
                lambda t: oracle.affine_matmul(x, t["codes"], t["scales"], t["biases"], 4, 64, t["bias"])[0]))
    qw, sw = oracle.quantize_int8_rows(w)
    out.append(("w8a8", N, {"w": qw, "scale_w": sw, "bias": bias},
                lambda t: oracle.w8a8_linear(x, t["w"], t["scale_w"], t["bias"])[0]))
    N4 = 96
    P4, s4 = oracle.pack_int4_cols(synth.normal(93, (K, N4), 0.02))
    out.append(("w4a8", N4, {"packed": P4, "scale_w": s4, "bias": None},
                lambda t: oracle.w4a8_linear(x, t["packed"], t["scale_w"], t["bias"])[0]))
    qg, sg = oracle.quantize_int8_groups(w, 128)
    out.append(("pergroup", N, {"w": qg, "scale_w": sg, "bias": bias},
                lambda t: oracle.pergroup_linear(x, t["w"], t["scale_w"], 128, t["bias"])[0]))
    NB = 72
    P = synth.any_bytes(94, NB // 4, K)
    out.append(("bitlinear", NB, {"packed": P, "bias": synth.normal(95, (NB,), 0.01)},
                lambda t: oracle.bitlinear(x, t["packed"], 4 * t["packed"].shape[0], 0.5, True, t["bias"])[0]))
    return out


def _rank(rank: int, world: int, port: int, q):
    sys.path.insert(0, ROOT)
    import datetime

    import torch
    import torch.distributed as dist

    import oracle
    from bit_quantized_linear_qmm_b200 import colsplit
    oracle.build()
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        results = []
        for fmt, N, weights, run in _layers():
            part = colsplit.shard(fmt, weights, N, world, rank)
            y_local = torch.from_numpy(np.ascontiguousarray(run(part)))
            y = colsplit.gather_y(y_local, fmt, N).numpy()
            results.append((fmt, bool(np.array_equal(y, run(weights)))))
        dist.barrier()
        q.put((rank, results))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_column_split_gathers_the_unsplit_layer(world):
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=240)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    for _ in range(world):
        rank, results = q.get()
        for fmt, ok in results:
            assert ok, (rank, fmt)


def test_blocks_cover_and_align():
    from bit_quantized_linear_qmm_b200 import colsplit
    for n, world, align in [(200, 2, 1), (96, 3, 16), (7, 4, 1), (4096, 8, 16)]:
        got = [colsplit.block(n, world, r, align) for r in range(world)]
        assert got[0][0] == 0 and got[-1][1] == n
        for (a0, a1), (b0, b1) in zip(got, got[1:]):
            assert a1 == b0 and a0 % align == 0
    idx = np.concatenate([colsplit.output_index("bitlinear", 72, 2, r) for r in range(2)])
    assert sorted(idx.tolist()) == list(range(72))

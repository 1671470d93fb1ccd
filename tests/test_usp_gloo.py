"""Unified sequence parallelism (Ulysses all-to-all x Ring) on CPU ranks over
gloo: the partition arithmetic of video_diffusion_transformer_02_b200.usp —
which tokens and heads each rank holds after the all-to-all, which key slice
each ring step attends, the positions handed to attention, the inverse
all-to-all — checked with the fp64 oracle as the per-shard attention and
join.  Every rank's output slice must equal the oracle's attention over the
whole sequence for those rows (to fp64 rounding)."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, U, R, mode, out):
    import datetime
    import sys
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        import seeded_inputs as si
        from video_diffusion_transformer_02_b200 import usp
        B, T, F, H, Hkv, d = 1, 8, 6, 4, 2, 16
        L = T * F
        q = si.normal_bf16(161, (B, L, H, d))
        k = si.normal_bf16(162, (B, L, Hkv, d))
        v = si.normal_bf16(163, (B, L, Hkv, d))
        kw = dict(mode=mode, F=F, chunk=2 if mode == "chunk_causal" else 1,
                  wb=1 if mode == "sliding" else 0)
        # rank (g, u): Ulysses group g = rank // U (sequence block g), member u
        g, u = rank // U, rank % U
        ugroups = [dist.new_group(list(range(gg * U, gg * U + U))) for gg in range(R)]
        rgroups = [dist.new_group([gg * U + uu for gg in range(R)]) for uu in range(U)]
        Ls = L // (U * R)
        tok0 = (g * U + u) * Ls
        as_t = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16))   # bf16 bits through the wires

        def attend(qs, ks, vs, q_tok0, k_tok0):
            o, lse = oracle.attention(qs.numpy().view(np.uint16), ks.numpy().view(np.uint16),
                                      vs.numpy().view(np.uint16), d ** -0.5, q_frame_offset=q_tok0 // F,
                                      k_frame_offset=k_tok0 // F, **kw)
            return torch.from_numpy(o), torch.from_numpy(lse)

        def merge(o_parts, lse_parts):
            Rn, Bn, Lq, h, dd = o_parts.shape
            op = o_parts.permute(0, 1, 3, 2, 4).reshape(Rn, -1, dd).numpy()
            lp = lse_parts.reshape(Rn, -1).numpy()
            o, _ = oracle.merge(op, lp)
            return torch.from_numpy(o).reshape(Bn, h, Lq, dd).permute(0, 2, 1, 3).contiguous()

        sl = slice(tok0, tok0 + Ls)
        o = usp.usp_attention(as_t(q[:, sl]), as_t(k[:, sl]), as_t(v[:, sl]), ugroups[g], rgroups[u], attend,
                              merge, tok0)
        ref, _ = oracle.attention(q, k, v, d ** -0.5, **kw)
        err = float(np.max(np.abs(o.numpy() - ref[:, sl])))
        out.put((rank, err, tuple(o.shape)))
    except Exception as e:   # report instead of leaving the parent waiting
        out.put((rank, repr(e), None))
        raise
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.parametrize("U,R", [(2, 1), (1, 2)], ids=["ulysses2", "ring2"])
@pytest.mark.parametrize("mode", ["full", "chunk_causal", "sliding"])
def test_usp_partition_two_ranks(U, R, mode):
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, U, R, mode, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((out.get(timeout=180) for _ in procs), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, err, shape in res:
        assert shape is not None, "rank %d failed: %s" % (rank, err)
        assert shape == (1, 24, 4, 16)
        assert err < 1e-12, "rank %d: max error %.3e against attention over the whole sequence" % (rank, err)

"""Context-parallel GDN scan on CPU ranks (gloo): the orchestration of
linear_attention_video_frame_b200.context_parallel -- frame split, one
all-gather of the interval composites, exclusive prefix, rescan -- run with
the oracle as its compute steps, against the oracle's single scan of the
whole clip.  (The CUDA kernels of the same steps are checked on the GPU in
tests/test_gpu_context_parallel.py.)"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleOps:
    """The three compute steps of the context-parallel scan, on the oracle
    (float64, CPU tensors)."""
    dtype = torch.float64

    def composite(self, k, v, alpha, beta, k_scale, out):
        import oracle
        B, H = k.shape[:2]
        for b in range(B):
            for h in range(H):
                T, U = oracle.gdn_interval_composite(k[b, h].numpy(), v[b, h].numpy(),
                                                     alpha[b, h].numpy(), beta[b, h].numpy(),
                                                     k_scale)
                out[0, b, h] = torch.from_numpy(T)
                out[1, b, h] = torch.from_numpy(U)
        return out

    def compose(self, gathered, state_in, state_out):
        import oracle
        n, _, B, H, D, _ = gathered.shape
        starts = torch.empty((n, B, H, D, D), dtype=torch.float64)
        for b in range(B):
            for h in range(H):
                comps = [(gathered[r, 0, b, h].numpy(), gathered[r, 1, b, h].numpy())
                         for r in range(n)]
                m0 = None if state_in is None else state_in[b, h].numpy()
                st = oracle.compose_exclusive_prefix(comps, m0)
                for r in range(n):
                    starts[r, b, h] = torch.from_numpy(st[r])
                if state_out is not None:
                    T, U = comps[-1]
                    state_out[b, h] = torch.from_numpy(T @ st[-1] + U)
        return starts

    def scan(self, q, k, v, alpha, beta, k_scale, state_in):
        import oracle
        o, _ = oracle.gdn_scan(q.numpy(), k.numpy(), v.numpy(), alpha.numpy(), beta.numpy(),
                               k_scale, state_in.numpy())
        return torch.from_numpy(o)


def _spec():
    import synth
    return synth.small(B=2, H=2, F=7, S=24, D=16, dtype="f32", seed=61)


def _clip():
    import synth
    spec = _spec()
    q, k, v = (torch.from_numpy(synth.full_values(spec, n).astype(np.float64)) for n in "qkv")
    a, bt = synth.gates(spec)
    m0, _ = synth.random_state(spec, 0.3)
    return spec, q, k, v, torch.from_numpy(a.astype(np.float64)), \
        torch.from_numpy(bt.astype(np.float64)), torch.from_numpy(m0.astype(np.float64))


def _rank(rank, world, port, q_out):
    import torch.distributed as dist
    from linear_attention_video_frame_b200.context_parallel import cp_scan_gdn, frame_interval
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        spec, q, k, v, a, bt, m0 = _clip()
        f0, f1 = frame_interval(spec.F, world, rank)
        sl = slice(f0, f1)
        so = torch.empty((spec.B, spec.H, spec.D, spec.D), dtype=torch.float64)
        o = cp_scan_gdn(q[:, :, sl].contiguous(), k[:, :, sl].contiguous(),
                        v[:, :, sl].contiguous(), a[:, :, sl].contiguous(),
                        bt[:, :, sl].contiguous(), spec.k_scale, state_in=m0, state_out=so,
                        ops=OracleOps())
        q_out.put((rank, f0, f1, o.numpy(), so.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3, 8])
def test_context_parallel_scan_equals_the_single_scan(world):
    import oracle
    ctx = mp.get_context("spawn")
    q_out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q_out)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q_out.get(timeout=180) for _ in range(world)), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    spec, q, k, v, a, bt, m0 = _clip()
    ref_o, ref_m = oracle.gdn_scan(q.numpy(), k.numpy(), v.numpy(), a.numpy(), bt.numpy(),
                                   spec.k_scale, m0.numpy())
    # the ranks' intervals tile the clip in order (world 8 > 7 frames: one rank is empty)
    assert [r[1] for r in res] == sorted(r[1] for r in res) and res[-1][2] == spec.F
    o = np.concatenate([r[3] for r in res], axis=2)
    scale = np.max(np.abs(ref_o))
    assert np.max(np.abs(o - ref_o)) <= 1e-10 * scale
    for r in res:      # every rank holds the state after the whole clip
        assert np.max(np.abs(r[4] - ref_m)) <= 1e-10 * np.max(np.abs(ref_m))


def test_frame_interval_tiles_the_clip():
    from linear_attention_video_frame_b200.context_parallel import frame_interval
    for F in (0, 1, 7, 181, 961):
        for world in (1, 2, 3, 8):
            spans = [frame_interval(F, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == F
            assert all(spans[i][1] == spans[i + 1][0] for i in range(world - 1))
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        frame_interval(10, 2, 2)

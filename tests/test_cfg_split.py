"""Host logic of the two-rank CFG split, on CPU with gloo (world size 2).

The forward and the Euler update are the oracle's (fp64, CPU tensors) so the
test runs without a GPU; what is checked is the split itself: which rank
takes which half, the order of the exchanged velocities, and that both ranks
end with the single-process result.  A swapped order would flip the sign of
the guidance term (g = 3.5) and fail.  Both exchange forms are covered: the
all-gather, and the peer form, where a file mapped by both processes stands
in for the IPC-mapped device buffer (handle = its path) and the slots
alternate per step behind one barrier.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as O
import synth
from helpers import draw_weights, tiny_config


def _free_port():
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def _problem():
    cfg = tiny_config()
    w = draw_weights(cfg, 501)
    x0 = synth.latents(502, (1, 4, 16, 16)).astype(np.float64)
    text = synth.text_embeddings(503, (2, 8, cfg.joint_attention_dim)).astype(np.float64)
    return cfg, w, x0, text, O.sigma_schedule(3, 1.73), [2, 8]


class _FileExchange:
    """The exchange buffer's host stand-in: two float64 slots in a file that
    the peer process maps (the 'IPC handle' is the file's path)."""

    def __init__(self, shape, out_dir, rank):
        self.path = os.path.join(out_dir, f"exchange{rank}.npy")
        self.arr = np.lib.format.open_memmap(self.path, mode="w+", dtype=np.float64, shape=(2,) + tuple(shape))
        self.peer_arr = None

    def handle(self):
        return self.path.encode()

    def open_peer(self, handle):
        self.peer_arr = np.lib.format.open_memmap(handle.decode(), mode="r")

    def local(self, slot):
        return torch.from_numpy(self.arr[slot])

    def peer(self, slot):
        return torch.from_numpy(np.array(self.peer_arr[slot]))

    def synchronize(self):
        self.arr.flush()


def _rank(rank, port, out_dir, use_lens, exchange):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=2)
    try:
        from diffusion_transformer_denoising_auraflow_b200.cfg_split import CFGSplitSampler
        cfg, w, x0, text, sig, lens = _problem()
        seen = []

        def fwd(lat, txt, t, vel, tl):
            seen.append(float(txt.double().sum()))
            v = O.transformer_forward(lat.numpy(), txt.numpy(), t.numpy(), w, cfg,
                                      text_len=None if tl is None else tl.numpy())
            vel.copy_(torch.from_numpy(v))

        def euler(lat, v, g, a, b):
            lat.copy_(torch.from_numpy(O.euler_cfg_step(lat.numpy(), v.numpy(), g, a, b)))

        def euler2(lat, vu, vc, g, a, b):
            v = np.concatenate([vu.numpy(), vc.numpy()])
            lat.copy_(torch.from_numpy(O.euler_cfg_step(lat.numpy(), v, g, a, b)))

        lat = torch.from_numpy(x0.copy())
        tl = torch.tensor(lens, dtype=torch.int32) if use_lens else None
        smp = CFGSplitSampler(None, None, lat, torch.from_numpy(text), sig, 3.5, text_len=tl, exchange=exchange,
                              _forward=fwd, _euler=euler, _euler2=euler2,
                              _make_exchange=lambda shape: _FileExchange(shape, out_dir, rank))
        for i in range(smp.n_steps):
            smp.step(i)
        np.save(os.path.join(out_dir, f"lat{rank}.npy"), lat.numpy())
        np.save(os.path.join(out_dir, f"seen{rank}.npy"), np.array(seen))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("exchange", ["peer", "nccl"])
@pytest.mark.parametrize("use_lens", [False, True])
def test_cfg_split_two_ranks_match_single_process(tmp_path, use_lens, exchange):
    mp.start_processes(_rank, args=(_free_port(), str(tmp_path), use_lens, exchange), nprocs=2, start_method="spawn")
    cfg, w, x0, text, sig, lens = _problem()
    x = x0.copy()
    for i in range(3):
        v = O.transformer_forward(np.concatenate([x, x]), text, np.full(2, sig[i]), w, cfg,
                                  text_len=lens if use_lens else None)
        x = O.euler_cfg_step(x, v, 3.5, sig[i], sig[i + 1])
    l0, l1 = np.load(tmp_path / "lat0.npy"), np.load(tmp_path / "lat1.npy")
    assert np.array_equal(l0, l1)                              # both ranks hold the same latents
    assert np.allclose(l0, x, rtol=1e-10, atol=1e-12)          # and the single-process result
    # rank 0 ran the uncond half, rank 1 the text half
    assert np.allclose(np.load(tmp_path / "seen0.npy"), text[0].sum())
    assert np.allclose(np.load(tmp_path / "seen1.npy"), text[1].sum())


def _rank_world3(rank, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=3)
    try:
        from diffusion_transformer_denoising_auraflow_b200.cfg_split import CFGSplitSampler
        try:
            CFGSplitSampler(None, None, torch.zeros(1, 4, 8, 8), torch.zeros(2, 4, 32), [1.0, 0.0], 3.5,
                            exchange="nccl")
            ok = False
        except ValueError:
            ok = True
        np.save(os.path.join(out_dir, f"ok{rank}.npy"), np.array(ok))
    finally:
        dist.destroy_process_group()


def test_cfg_split_needs_two_ranks(tmp_path):
    mp.start_processes(_rank_world3, args=(_free_port(), str(tmp_path)), nprocs=3, start_method="spawn")
    for r in range(3):
        assert bool(np.load(tmp_path / f"ok{r}.npy"))

"""The fused CFG exchange on a GPU: two processes, one per CFG half.

Each process runs the forward of its half of the CFG batch into its exchange
buffer, the processes meet at one host barrier per step (gloo), and each
applies the guidance + Euler update reading its own half and the other
process's half through the CUDA IPC mapping (af_exchange_*,
af_euler_cfg_step2).  Here both processes share one GPU, so the peer mapping
points at the same device's memory; across two GPUs the same loads would
cross NVLink.  No kernel waits on the other process: ordering is the stream
sync and the host barrier.

Every forward is batch-independent bit for bit and the update does the same
arithmetic as af_euler_cfg_step, so after three steps both processes must
hold exactly the latents of the single-process loop (af_denoise_step on the
CFG batch of 2).
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
from helpers import af_config, draw_weights, tiny_config, to_bf16, to_f32, upload

pytestmark = pytest.mark.gpu

SEED = 601


def _free_port():
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def _sigmas():
    return [float(np.float32(x)) for x in O.sigma_schedule(3, 1.73)]


def _rank(rank, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=2)
    try:
        torch.cuda.set_device(0)
        import diffusion_transformer_denoising_auraflow_b200 as af
        from diffusion_transformer_denoising_auraflow_b200.cfg_split import CFGSplitSampler
        cfg = tiny_config()
        w = af.Weights(af_config(cfg))
        upload(w, draw_weights(cfg, SEED))
        s = af.Scratch(w, 1, 64, 8)
        lat = to_f32(synth.latents(SEED + 1, (1, 4, 16, 16)))
        text = to_bf16(synth.text_embeddings(SEED + 2, (2, 8, cfg.joint_attention_dim)))
        smp = CFGSplitSampler(w, s, lat, text, _sigmas(), 3.5, exchange="peer")
        for i in range(smp.n_steps):
            smp.step(i)
        torch.cuda.synchronize()
        np.save(os.path.join(out_dir, f"lat{rank}.npy"), lat.cpu().numpy())
        dist.barrier()          # the peer is done reading this process's buffer
        smp.close()
        s.close()
        w.close()
    finally:
        dist.destroy_process_group()


def test_cfg_split_peer_exchange_two_processes(tmp_path):
    mp.start_processes(_rank, args=(_free_port(), str(tmp_path)), nprocs=2, start_method="spawn")
    import diffusion_transformer_denoising_auraflow_b200 as af
    cfg = tiny_config()
    w = af.Weights(af_config(cfg))
    upload(w, draw_weights(cfg, SEED))
    s = af.Scratch(w, 2, 64, 8)
    lat = to_f32(synth.latents(SEED + 1, (1, 4, 16, 16)))
    text = to_bf16(synth.text_embeddings(SEED + 2, (2, 8, cfg.joint_attention_dim)))
    sig = _sigmas()
    for i in range(3):
        af.denoise_step(w, s, lat, text, 3.5, sig[i], sig[i + 1])
    s.sync()
    ref = lat.cpu().numpy()
    l0, l1 = np.load(tmp_path / "lat0.npy"), np.load(tmp_path / "lat1.npy")
    assert np.array_equal(l0, l1)
    assert np.array_equal(l0, ref)
    assert np.abs(ref - synth.latents(SEED + 1, (1, 4, 16, 16))).max() > 0   # the steps moved the latent

"""muon_step_batched_host_grad: gradients in pinned host memory, streamed in chunk by chunk
while earlier chunks compute.  Every matrix goes through the same kernels with the same
per-matrix arithmetic as muon_step_batched, so W and M must come out bit-identical."""
import ctypes

import numpy as np
import pytest
import torch

from matrix_orthogonalising_optimizer_02_b200 import binding as mb

pytestmark = pytest.mark.gpu

SHAPES = [(256, 512), (512, 256), (384, 384), (128, 1024), (1024, 128), (256, 256), (512, 512), (640, 384),
          (384, 640), (256, 768), (768, 256), (128, 128)]


def _set(seed, g_f32=(1, 7)):
    gen = torch.Generator(device="cuda")
    gen.manual_seed(seed)
    mats = []
    for i, (r, c) in enumerate(SHAPES):
        W = torch.empty((r, c), device="cuda").normal_(0, 0.02, generator=gen).to(torch.bfloat16)
        gdt = torch.float32 if i in g_f32 else torch.bfloat16
        G = torch.empty((r, c), device="cuda").normal_(0, 1e-3, generator=gen).to(gdt)
        M = torch.empty((r, c), device="cuda").normal_(0, 1e-3, generator=gen)
        mats.append(mb.Matrix(W, G, M))
    return mats


def test_host_gradient_step_is_bit_identical_to_device_step():
    hp = mb.hyper(lr=0.02, beta=0.95, weight_decay=0.1, nesterov=True)
    dev = _set(31)
    host = [mb.Matrix(m.W.clone(), m.G.cpu().pin_memory(), m.M.clone()) for m in dev]
    ws_d = mb.workspace(mb.muon_step_workspace_size(dev, hp))
    ws_h = mb.workspace(mb.muon_step_host_grad_workspace_size(host, hp))
    gen = torch.Generator(device="cuda")
    gen.manual_seed(32)
    for step in range(3):
        if step:
            for d, h in zip(dev, host):
                d.G.copy_(torch.empty(d.G.shape, device="cuda").normal_(0, 1e-3, generator=gen).to(d.G.dtype))
                h.G.copy_(d.G.cpu())
        mb.muon_step_batched(dev, hp, ws_d)
        mb.muon_step_batched_host_grad(host, hp, ws_h)
        assert mb.device_status(ws_d) == mb.MUON_OK
        assert mb.device_status(ws_h) == mb.MUON_OK
        for d, h in zip(dev, host):
            assert torch.equal(d.W, h.W) and torch.equal(d.M, h.M)


def test_host_gradient_step_rejects_pageable_gradients():
    hp = mb.hyper(lr=0.02)
    dev = _set(33, g_f32=())
    host = [mb.Matrix(m.W, m.G.cpu().pin_memory(), m.M) for m in dev]
    ws = mb.workspace(mb.muon_step_host_grad_workspace_size(host, hp))
    pageable = np.zeros(SHAPES[0], dtype=np.uint16)
    descs = mb._descs(host, g_on_host=True)
    descs[0].G = pageable.ctypes.data
    lib = mb.load()
    st = lib.muon_step_batched_host_grad(descs, len(host), ctypes.byref(hp[0]), ws.data_ptr(),
                                         ws.numel() * ws.element_size(), None)
    assert st == mb.MUON_ERR_INVALID_ARG
    with pytest.raises(ValueError):
        mb.muon_step_batched_host_grad([mb.Matrix(dev[0].W, dev[0].G.cpu(), dev[0].M)], hp, ws)

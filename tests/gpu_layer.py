"""Test helper: one weight matrix held on the GPU through the C ABI, fed with the
same seeded inputs as an oracle LayerState."""
from ctypes import byref, c_void_p

import numpy as np
import torch

import oracle as O
import quantized_rank_gradient_b200 as qg


def round_up(x, a):
    return -(-x // a) * a


def stream():
    return c_void_p(torch.cuda.current_stream().cuda_stream)


def lib_config(oc: O.Config):
    return qg.config(oc.m, oc.n, oc.r, beta1=oc.beta1, beta2=oc.beta2, eps=oc.eps, lr=oc.lr, alpha=oc.alpha,
                     gamma=oc.gamma, delta0=oc.delta0, oversample=oc.oversample, power_iters=oc.power_iters,
                     seed=oc.seed, layer_id=oc.layer_id, mom_refresh=oc.mom_refresh, proj_side=oc.proj_side,
                     w_rescale=oc.w_rescale)


def upload_gradient(G_bits: np.ndarray, device="cuda"):
    """bf16 bit patterns (m x n uint16) -> device int16 tensor m x ldg (ldg % 8 == 0)."""
    m, n = G_bits.shape
    ldg = round_up(n, 8)
    g = torch.zeros((m, ldg), dtype=torch.int16)
    g[:, :n] = torch.from_numpy(G_bits.view(np.int16))
    return g.to(device), ldg


class GpuLayer:
    def __init__(self, oc: O.Config, Wq: np.ndarray, sW: np.ndarray, device="cuda"):
        self.oc = oc
        self.cfg = lib_config(oc)
        m, n = oc.m, oc.n
        self.ldw = round_up(n, 16)
        self.W = torch.zeros((m, self.ldw), dtype=torch.int8, device=device)
        self.W[:, :n] = torch.from_numpy(np.asarray(Wq, np.int8)).to(device)
        self.sW = torch.from_numpy(np.asarray(sW, np.float32)).to(device)
        nbytes = qg.qg_state_bytes(byref(self.cfg))
        assert nbytes > 0
        self.state = torch.zeros(nbytes, dtype=torch.uint8, device=device)
        self.h = c_void_p()
        qg.check(qg.qg_layer_init(byref(self.h), byref(self.cfg), self.state.data_ptr(), nbytes, self.W.data_ptr(),
                                  self.ldw, self.sW.data_ptr(), stream()), "qg_layer_init")
        self.v = qg.qg_layer_views()
        qg.check(qg.qg_layer_views_get(self.h, byref(self.v)))
        self.ws = torch.zeros(qg.qg_step_workspace_bytes(byref(self.cfg)), dtype=torch.uint8, device=device)
        self.device = device

    def close(self):
        if self.h:
            qg.qg_layer_destroy(self.h)
            self.h = c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def set_projection(self, Pq: np.ndarray, sP: np.ndarray, keep_prev=0):
        a = torch.from_numpy(np.ascontiguousarray(Pq, np.uint8)).to(self.device)
        b = torch.from_numpy(np.ascontiguousarray(sP, np.float32)).to(self.device)
        qg.check(qg.qg_layer_set_projection(self.h, a.data_ptr(), b.data_ptr(), keep_prev, stream()))
        torch.cuda.synchronize()

    def step(self, G_dev: torch.Tensor, ldg: int):
        qg.check(qg.qg_step(self.h, G_dev.data_ptr(), ldg, self.ws.data_ptr(), self.ws.numel(), stream()), "qg_step")

    def region(self, ptr, nbytes):
        off = ptr - self.state.data_ptr()
        assert 0 <= off and off + nbytes <= self.state.numel()
        return self.state[off: off + nbytes]

    def weights(self) -> np.ndarray:
        return self.W[:, : self.oc.n].cpu().numpy()

    def moments(self):
        rows, cols = self.v.mom_rows, self.v.mom_cols
        ld, nb = self.v.ld_mom, self.v.nblk
        Mq = self.region(self.v.Mq, rows * ld).view(torch.int8).view(rows, ld)[:, :cols].cpu().numpy()
        Vq = self.region(self.v.Vq, rows * ld).view(torch.int8).view(rows, ld)[:, :cols].cpu().numpy()
        sM = self.region(self.v.sM, rows * nb * 4).view(torch.float32).view(rows, nb).cpu().numpy()
        sV = self.region(self.v.sV, rows * nb * 4).view(torch.float32).view(rows, nb).cpu().numpy()
        return Mq, sM, Vq, sV

    def projection(self):
        mr = self.v.p_rows * self.oc.r
        Pq = self.region(self.v.Pq, (mr + 1) // 2).cpu().numpy()
        sP = self.region(self.v.sP, -(-mr // 64) * 4).view(torch.float32).cpu().numpy()
        return Pq, sP

    def scratch_N(self):
        """N (R's shape, bf16 bits) from the step workspace (layout: P~ then N, 256-aligned)."""
        p, r = self.v.p_rows, self.oc.r
        rows, cols = self.v.mom_rows, self.v.mom_cols
        off = round_up(p * r * 2, 256)
        ldN = round_up(cols, 32)
        return (self.ws[off: off + rows * ldN * 2].view(torch.int16).view(rows, ldN)[:, :cols].cpu().numpy()
                .view(np.uint16))

    def refresh(self, G_dev: torch.Tensor, ldg: int, force=0):
        """qg_refresh; returns (info, float32 projection from the workspace)."""
        if not hasattr(self, "rws"):
            self.rws = torch.zeros(qg.qg_refresh_workspace_bytes(byref(self.cfg)), dtype=torch.uint8,
                                   device=self.device)
        info = qg.qg_refresh_info()
        qg.check(qg.qg_refresh(self.h, G_dev.data_ptr(), ldg, force, self.rws.data_ptr(), self.rws.numel(),
                               byref(info), stream()), "qg_refresh")
        torch.cuda.synchronize()
        p, r = self.v.p_rows, self.oc.r
        P = self.rws[: p * r * 4].view(torch.float32).view(p, r).cpu().numpy().copy()
        return info, P

    def status(self):
        return qg.qg_layer_status(self.h, stream())

    def sched(self):
        s = qg.qg_sched()
        qg.check(qg.qg_layer_sched_get(self.h, byref(s)))
        return s

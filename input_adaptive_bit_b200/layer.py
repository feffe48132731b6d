"""Device-memory holder for one GRINQH linear layer (PyTorch plumbing only).

``GrinqhLinear`` packs the layer's base codes once with ``grinqh_pack`` and
keeps the buffers that ``grinqh_assign`` and ``grinqh_gemv`` write, so a
decode step is two library calls on caller-owned memory.  torch allocates the
memory and provides the stream; all arithmetic runs in libgrinqh.
"""
from __future__ import annotations

import torch

from . import (MAX_GROUP, grinqh_decode_gemv_group, grinqh_group_workspace_bytes,
               grinqh_assign, grinqh_decode_gemv, grinqh_gemv, grinqh_gemv_dense4, grinqh_pack,
               grinqh_pack_dense4, grinqh_dense4_workspace_bytes, grinqh_prefill_gemm,
               grinqh_prefill_workspace_bytes, grinqh_workspace_bytes)

GROUP = 128


def _dev(t, device, dtype):
    t = torch.as_tensor(t)
    if t.dtype != dtype:
        raise TypeError(f"expected {dtype}, got {t.dtype}")
    return t.to(device=device).contiguous()


class GrinqhLinear:
    """One decode GEMV y = W_hat^T x of GRINQH.

    q: uint8 [d_in, d_out] base codes (< 2^b_max); s, z: fp16 [d_in/128, d_out].
    """

    def __init__(self, q, s, z, b_max: int, device="cuda", stream=None):
        self.device = torch.device(device)
        q = _dev(q, self.device, torch.uint8)
        self.d_in, self.d_out = int(q.shape[0]), int(q.shape[1])
        self.b_max = int(b_max)
        self.P = self.b_max // 2
        self.G = self.d_in // GROUP
        self.s = _dev(s, self.device, torch.float16)
        self.z = _dev(z, self.device, torch.float16)
        self.planes = torch.empty((self.d_in, self.P, self.d_out // 16), dtype=torch.int32,
                                  device=self.device)
        grinqh_pack(q, self.d_in, self.d_out, self.b_max, self.planes, stream)
        del q
        # per-call buffers
        self.b = torch.empty(self.d_in, dtype=torch.uint8, device=self.device)
        self.lists = torch.empty((self.P, self.d_in), dtype=torch.int32, device=self.device)
        self.counts = torch.empty(self.P, dtype=torch.int32, device=self.device)
        self.grp_sums = torch.empty((2, self.G), dtype=torch.float32, device=self.device)
        self.ws_bytes = grinqh_workspace_bytes(self.d_in, self.d_out, self.b_max)
        self.ws = torch.zeros(self.ws_bytes, dtype=torch.uint8, device=self.device)
        self.y = torch.empty(self.d_out, dtype=torch.float32, device=self.device)
        self.prefill_ws_bytes = grinqh_prefill_workspace_bytes()
        self.prefill_ws = torch.zeros(max(self.prefill_ws_bytes, 256), dtype=torch.uint8,
                                      device=self.device)

    def assign(self, x, theta, phi=None, stream=None):
        grinqh_assign(x, theta, self.d_in, self.b_max, phi, self.b, self.lists, self.counts,
                      self.grp_sums, self.ws, self.ws_bytes, stream)

    def gemv(self, y=None, stream=None):
        y = self.y if y is None else y
        grinqh_gemv(self.planes, self.s, self.z, self.grp_sums, self.d_in, self.d_out,
                    self.b_max, y, self.ws, self.ws_bytes, stream)
        return y

    def decode(self, x, theta, phi=None, y=None, outputs=True, stream=None):
        """The fused single-kernel decode step; with outputs=True it also fills
        b, lists, counts and grp_sums as grinqh_assign would."""
        y = self.y if y is None else y
        o = outputs
        grinqh_decode_gemv(self.planes, self.s, self.z, x, theta, phi, self.d_in, self.d_out,
                           self.b_max, y, self.b if o else None, self.lists if o else None,
                           self.counts if o else None, self.grp_sums if o else None, self.ws,
                           self.ws_bytes, stream)
        return y

    def prefill(self, X, phi=None, Y=None, stream=None):
        """Y[T][d_out] (fp32) = X[T][d_in] (fp16) times W_hat at the full width b_max:
        the prefill GEMM on the same packed planes."""
        T = int(X.shape[0])
        if Y is None:
            Y = torch.empty((T, self.d_out), dtype=torch.float32, device=self.device)
        grinqh_prefill_gemm(self.planes, self.s, self.z, X, phi, T, self.d_in, self.d_out,
                            self.b_max, Y, self.prefill_ws, self.prefill_ws_bytes, stream)
        return Y

    def __call__(self, x, theta, phi=None, y=None, stream=None):
        """x: fp16 [d_in] on the device; theta: fp32 [b_max/2] on the device."""
        self.assign(x, theta, phi, stream)
        return self.gemv(y, stream)


class DecodeGroup:
    """Independent GrinqhLinear layers (q, k, v of a decoder layer; gate, up) decoded in
    one launch of grinqh_decode_gemv_group; holds the group's workspace."""

    def __init__(self, layers, device="cuda"):
        if not 1 <= len(layers) <= MAX_GROUP:
            raise ValueError(f"a group holds 1..{MAX_GROUP} layers, got {len(layers)}")
        self.layers = list(layers)
        self.ws_bytes = grinqh_group_workspace_bytes()
        self.ws = torch.zeros(self.ws_bytes, dtype=torch.uint8, device=torch.device(device))

    def __call__(self, xs, thetas, phis=None, ys=None, stream=None):
        """xs, thetas (and phis, ys if given): one per layer; returns the ys."""
        phis = phis or [None] * len(self.layers)
        ys = ys or [lin.y for lin in self.layers]
        grinqh_decode_gemv_group(
            [(lin.planes, lin.s, lin.z, x, th, ph, lin.d_in, lin.d_out, lin.b_max, y)
             for lin, x, th, ph, y in zip(self.layers, xs, thetas, phis, ys)],
            self.ws, self.ws_bytes, stream)
        return ys


class Dense4Linear:
    """The in-library dense 4-bit comparator on the same shape."""

    def __init__(self, q4, s, z, device="cuda", stream=None):
        self.device = torch.device(device)
        q4 = _dev(q4, self.device, torch.uint8)
        self.d_in, self.d_out = int(q4.shape[0]), int(q4.shape[1])
        self.s = _dev(s, self.device, torch.float16)
        self.z = _dev(z, self.device, torch.float16)
        self.w4 = torch.empty((self.d_in, self.d_out // 8), dtype=torch.int32, device=self.device)
        grinqh_pack_dense4(q4, self.d_in, self.d_out, self.w4, stream)
        self.ws_bytes = grinqh_dense4_workspace_bytes(self.d_in, self.d_out)
        self.ws = torch.zeros(max(self.ws_bytes, 256), dtype=torch.uint8, device=self.device)
        self.y = torch.empty(self.d_out, dtype=torch.float32, device=self.device)

    def __call__(self, x, y=None, stream=None):
        y = self.y if y is None else y
        grinqh_gemv_dense4(self.w4, self.s, self.z, x, self.d_in, self.d_out, y, self.ws,
                           self.ws_bytes, stream)
        return y

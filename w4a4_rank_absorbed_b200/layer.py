"""SVDQLinear: a packed SVDQuant W4A4 linear layer on one B200.

Holds the packed residual weight and the low-rank factors in device memory
and runs the forward pass as two launches of the CUDA library
(SVDQuant review §4.3: down-projection fused into the quantization kernel,
up-projection fused into the 4-bit GEMM):

    svdq_quantize_act   X (bf16)  ->  Xq, SFx, LAs
    svdq_linear         Xq, SFx, Wq, SFw, LAs, L2p, bias  ->  Y

torch is used for device memory and streams only.
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np
import torch

from . import svdq as _C
from .calib import LayerData


def _f32(x) -> float:
    return float(np.float32(x))


def check_device(t: Optional[torch.Tensor], device: torch.device, name: str) -> None:
    """Raise ValueError unless tensor `t` (when given) lives on `device`.

    The library launches on the calling thread's current device with raw pointers; a tensor on
    another GPU would be read through a pointer that device cannot resolve."""
    if t is None:
        return
    want = torch.device(device)
    if t.device.type != want.type or (want.index is not None and t.device.index != want.index):
        raise ValueError(f"{name} is on {t.device}, the layer on {want}")


class SVDQLinear:
    def __init__(self, data: LayerData, device: Optional[torch.device] = None, stream=None):
        dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.device = dev
        self.K, self.N, self.r = data.K, data.N, data.r
        self.gs_x = _f32(data.gs_x)
        K, N, r = self.K, self.N, self.r
        with torch.cuda.device(dev):
            R = data.R.to(dev, torch.float32).contiguous()
            L2b = data.L2b.to(dev).contiguous() if r else None
            self.Wq = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
            self.SFw = torch.empty(_C.svdq_sf_bytes(N, K), dtype=torch.uint8, device=dev)
            self.gs_w_dev = torch.empty(1, dtype=torch.float32, device=dev)
            self.L2p = torch.empty((N, r), dtype=torch.bfloat16, device=dev) if r else None
            # The packing stream may differ from torch's current stream: the staging tensors are
            # produced on the current stream, so the packing waits for it; the library writes gs_w
            # to host memory after synchronising the packing stream, so R and L2b are no longer
            # read when they are freed below.
            if stream is not None:
                ps = stream if isinstance(stream, torch.cuda.Stream) else \
                    torch.cuda.ExternalStream(_C.stream_handle(stream), device=dev)
                ps.wait_stream(torch.cuda.current_stream(dev))
            self.gs_w = _f32(_C.svdq_pack_weight(R, L2b, K, N, r, self.Wq, self.SFw, self.gs_w_dev, self.L2p,
                                                 stream, sync=True))
            del R, L2b
            self.inv_s = data.inv_s.to(dev, torch.float32).contiguous()
            self.L1fT = data.L1fT.to(dev).contiguous() if r else None
            self.bias = data.bias.to(dev).contiguous() if data.bias is not None else None
        self.lr_scale = _f32(1.0 / (np.float64(self.gs_x) * np.float64(self.gs_w)))
        self._act: Dict[int, tuple] = {}

    # ------------------------------------------------------------ checkpoint --
    _PACKED = ("Wq", "SFw", "gs_w_dev", "L2p", "inv_s", "L1fT", "bias")

    def state_dict(self) -> Dict[str, object]:
        """The packed layer as plain tensors (host copies) and scalars: save it with torch.save and
        rebuild with SVDQLinear.from_state_dict without packing the weight again."""
        out: Dict[str, object] = {"K": self.K, "N": self.N, "r": self.r, "gs_x": self.gs_x, "gs_w": self.gs_w,
                                  "lr_scale": self.lr_scale}
        for k in self._PACKED:
            t = getattr(self, k)
            out[k] = None if t is None else t.detach().cpu()
        return out

    @classmethod
    def from_state_dict(cls, state: Dict[str, object], device: Optional[torch.device] = None) -> "SVDQLinear":
        """A layer from state_dict() output, its buffers copied to `device` (no packing kernel runs)."""
        self = cls.__new__(cls)
        dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.device = dev
        self.K, self.N, self.r = int(state["K"]), int(state["N"]), int(state["r"])
        self.gs_x, self.gs_w, self.lr_scale = float(state["gs_x"]), float(state["gs_w"]), float(state["lr_scale"])
        for k in cls._PACKED:
            t = state[k]
            setattr(self, k, None if t is None else t.to(dev).contiguous())
        expect = {"Wq": (self.N, self.K // 2), "L2p": (self.N, self.r) if self.r else None,
                  "inv_s": (self.K,), "L1fT": (self.r, self.K) if self.r else None}
        for k, shape in expect.items():
            t = getattr(self, k)
            if (shape is None) != (t is None) or (t is not None and tuple(t.shape) != shape):
                raise ValueError(f"state entry {k} has shape {None if t is None else tuple(t.shape)}, expected {shape}")
        if self.SFw.numel() != _C.svdq_sf_bytes(self.N, self.K):
            raise ValueError("state entry SFw has the wrong size")
        self._act = {}
        return self

    def act_buffers(self, M: int):
        """Device buffers of the quantized activations for M rows (allocated once per M): Xq, SFx, LAs."""
        return self._act_set(M)[:3]

    def _act_set(self, M: int):
        if M not in self._act:
            K, r, dev = self.K, self.r, self.device
            with torch.cuda.device(dev):
                self._act[M] = (torch.empty((M, K // 2), dtype=torch.uint8, device=dev),
                                torch.empty(_C.svdq_sf_bytes(M, K), dtype=torch.uint8, device=dev),
                                torch.empty((M, 2 * r), dtype=torch.bfloat16, device=dev) if r else None,
                                _C.new_workspace(M, K, r, dev))
        return self._act[M]

    def quantize(self, X: torch.Tensor, stream=None):
        check_device(X, self.device, "X")
        M = X.shape[0]
        Xq, SFx, LAs, ws = self._act_set(M)
        with torch.cuda.device(self.device):
            _C.svdq_quantize_act(X, M, self.K, self.inv_s, self.gs_x, self.L1fT, self.r, self.lr_scale,
                                 Xq, SFx, LAs, ws, stream)
        return Xq, SFx, LAs

    def gemm(self, Xq, SFx, LAs, Y: torch.Tensor, stream=None):
        for t, name in ((Xq, "Xq"), (SFx, "SFx"), (LAs, "LAs"), (Y, "Y")):
            check_device(t, self.device, name)
        M = Xq.shape[0]
        with torch.cuda.device(self.device):
            _C.svdq_linear(Xq, SFx, self.gs_x, self.Wq, self.SFw, self.gs_w, LAs, self.L2p, self.r, self.bias,
                           Y, 1 if Y.dtype == torch.float32 else 0, M, self.N, self.K, stream)
        return Y

    def gemm_gelu_quantize(self, Xq, SFx, LAs, nxt: "SVDQLinear", stream=None):
        """This layer's GEMM with GELU and `nxt`'s activation quantization in its epilogue (no Y is
        written); returns nxt's quantized activations (Xq2, SFx2, LAs2), ready for nxt.gemm."""
        for t, name in ((Xq, "Xq"), (SFx, "SFx"), (LAs, "LAs")):
            check_device(t, self.device, name)
        if nxt.device != self.device or nxt.K != self.N:
            raise ValueError("the next layer must be on the same device and take this layer's N as its K")
        M = Xq.shape[0]
        Xq2, SFx2, LAs2 = nxt.act_buffers(M)
        key = ("gq", M, nxt.r)
        if key not in self._act:
            self._act[key] = _C.new_gelu_quantize_workspace(M, self.N, nxt.r, self.device)
        with torch.cuda.device(self.device):
            _C.svdq_linear_gelu_quantize(Xq, SFx, self.gs_x, self.Wq, self.SFw, self.gs_w, LAs, self.L2p, self.r,
                                         self.bias, M, self.N, self.K, nxt.inv_s, nxt.gs_x, nxt.L1fT, nxt.r,
                                         nxt.lr_scale, Xq2, SFx2, LAs2, self._act[key], stream)
        return Xq2, SFx2, LAs2

    def forward(self, X: torch.Tensor, out: Optional[torch.Tensor] = None, y_fp32: bool = False,
                stream=None) -> torch.Tensor:
        """Y = layer(X); X bf16 [M, K] on the device; returns bf16 (or fp32) [M, N]."""
        if X.dtype != torch.bfloat16 or X.dim() != 2 or X.shape[1] != self.K:
            raise ValueError("X must be bf16 [M, K]")
        check_device(X, self.device, "X")
        check_device(out, self.device, "out")
        M = X.shape[0]
        if out is None:
            out = torch.empty((M, self.N), dtype=torch.float32 if y_fp32 else torch.bfloat16, device=self.device)
        Xq, SFx, LAs = self.quantize(X, stream)
        return self.gemm(Xq, SFx, LAs, out, stream)

    __call__ = forward

    def forward_host(self, X_host: torch.Tensor, Y_host: torch.Tensor, X_dev: torch.Tensor,
                     Y_dev: torch.Tensor) -> None:
        """End-to-end call with host buffers: H2D of X, the two kernels, D2H of Y (asynchronous)."""
        X_dev.copy_(X_host, non_blocking=True)
        self.forward(X_dev, out=Y_dev)
        Y_host.copy_(Y_dev, non_blocking=True)

    def forward_host_stream(self, X_hosts, Y_hosts, X_devs, Y_devs) -> None:
        """A sequence of host batches through the layer, copies overlapped with compute.

        Batch i: its X (pinned host) is copied in on one stream, the two kernels run on a second,
        its Y is copied out (to pinned host) on a third, so batch i+1's copy in and batch i-1's
        copy out overlap batch i's kernels.  X_devs / Y_devs are two (or more) device buffers used
        in turn; a buffer is refilled only after the batch that used it has left it.  Asynchronous
        with respect to the host; events order the streams.
        """
        nb = len(X_devs)
        cur = torch.cuda.current_stream(self.device)
        s_in, s_cmp, s_out = (torch.cuda.Stream(device=self.device) for _ in range(3))
        for st in (s_in, s_cmp, s_out):
            st.wait_stream(cur)
        done_cmp = [None] * nb
        done_out = [None] * nb
        for i, (Xh, Yh) in enumerate(zip(X_hosts, Y_hosts)):
            b = i % nb
            with torch.cuda.stream(s_in):
                if done_cmp[b] is not None:
                    s_in.wait_event(done_cmp[b])          # the kernels that read X_devs[b] are done
                X_devs[b].copy_(Xh, non_blocking=True)
                ev_in = torch.cuda.Event()
                ev_in.record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(ev_in)
                if done_out[b] is not None:
                    s_cmp.wait_event(done_out[b])         # Y_devs[b] has been copied out
                self.forward(X_devs[b], out=Y_devs[b], stream=s_cmp)
                done_cmp[b] = torch.cuda.Event()
                done_cmp[b].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(done_cmp[b])
                Yh.copy_(Y_devs[b], non_blocking=True)
                done_out[b] = torch.cuda.Event()
                done_out[b].record(s_out)
        for st in (s_in, s_cmp, s_out):
            cur.wait_stream(st)


class SVDQMLP:
    """Two SVDQuant layers with GELU (tanh form) between them, fc2(GELU(fc1(X))).

    fused=True (the default): three launches of the library per call plus the small reduction of
    fc2's down-projection: fc1's activation kernel, fc1's GEMM whose epilogue applies GELU and
    quantizes the result as fc2's activations (svdq_linear_gelu_quantize), fc2's GEMM.  fused=False
    runs the unfused pair: fc1's layer, svdq_gelu_bf16, fc2's layer (fc1's output makes a round trip
    through memory as bf16)."""

    def __init__(self, fc1: SVDQLinear, fc2: SVDQLinear):
        if fc2.K != fc1.N or fc2.device != fc1.device:
            raise ValueError("fc2 must take fc1's output on the same device")
        self.fc1, self.fc2 = fc1, fc2
        self._mid: Dict[int, torch.Tensor] = {}

    def forward(self, X: torch.Tensor, out: Optional[torch.Tensor] = None, fused: bool = True,
                stream=None) -> torch.Tensor:
        fc1, fc2 = self.fc1, self.fc2
        M = X.shape[0]
        if out is None:
            out = torch.empty((M, fc2.N), dtype=torch.bfloat16, device=fc1.device)
        check_device(out, fc1.device, "out")
        if fused:
            Xq, SFx, LAs = fc1.quantize(X, stream)
            return fc2.gemm(*fc1.gemm_gelu_quantize(Xq, SFx, LAs, fc2, stream), out, stream)
        if M not in self._mid:
            self._mid[M] = (torch.empty((M, fc1.N), dtype=torch.bfloat16, device=fc1.device),
                            torch.empty((M, fc1.N), dtype=torch.bfloat16, device=fc1.device))
        Y1, X2 = self._mid[M]
        fc1.forward(X, out=Y1, stream=stream)
        with torch.cuda.device(fc1.device):
            _C.svdq_gelu_bf16(Y1, Y1.numel(), X2, stream)
        return fc2.forward(X2, out=out, stream=stream)

    __call__ = forward

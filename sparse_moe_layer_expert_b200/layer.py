"""MoeLayer: device-resident weights, bias, workspace and error flag of one
FP8 DeepSeekMoE layer, with forward / bias-update calls into libmoefp8.

Plumbing only: torch allocates the buffers; quantization, routing, the
grouped GEMMs and the combine all run in the library's kernels.
"""
from __future__ import annotations

import torch

from . import _binding as B


class MoeLayer:
    def __init__(self, shape: dict, device="cuda"):
        """shape: dict with H, I, Nr, Kr and optionally Ns (1), n_groups,
        topk_groups, route_scale."""
        self.shape = dict(shape)
        self.cfg = B.config_from(shape)
        c = self.cfg
        self.E = c.n_routed + c.n_shared
        H, I = c.hidden, c.inter
        dev = torch.device(device)
        self.device = dev
        self.w13 = torch.empty((self.E, 2 * I, H), dtype=torch.uint8, device=dev)
        self.s13 = torch.empty((self.E, 2 * I // 128, H // 128), dtype=torch.float32, device=dev)
        self.w2 = torch.empty((self.E, H, I), dtype=torch.uint8, device=dev)
        self.s2 = torch.empty((self.E, H // 128, I // 128), dtype=torch.float32, device=dev)
        self.wr = torch.empty((c.n_routed, H), dtype=torch.bfloat16, device=dev)
        self.bias = torch.zeros((c.n_routed,), dtype=torch.float32, device=dev)
        self.err = B.new_err_flag(dev)
        self._ws: dict[int, torch.Tensor] = {}

    # -------------------------------------------------------------- weights
    def set_expert(self, e: int, w13_bf16: torch.Tensor, w2_bf16: torch.Tensor, stream=None) -> None:
        """Quantize expert e's bf16 weights (128x128 blocks) into place, with
        the scale rule of the layer's scale mode."""
        pow2 = self.cfg.scale_mode == B.MOE_SCALE_POW2
        B.fp8_quant_128x128(w13_bf16.contiguous(), q=self.w13[e], scales=self.s13[e], stream=stream, pow2=pow2)
        B.fp8_quant_128x128(w2_bf16.contiguous(), q=self.w2[e], scales=self.s2[e], stream=stream, pow2=pow2)

    def set_router(self, wr_bf16: torch.Tensor, bias: torch.Tensor) -> None:
        self.wr.copy_(wr_bf16)
        self.bias.copy_(bias)

    @classmethod
    def from_generator(cls, shape: dict, expert_fn, wr: torch.Tensor, bias: torch.Tensor, device="cuda"):
        """expert_fn(e) -> (w13 bf16 [2I, H], w2 bf16 [H, I]) on `device`,
        called once per expert (routed 0..Nr-1, then shared)."""
        layer = cls(shape, device)
        for e in range(layer.E):
            w13, w2 = expert_fn(e)
            layer.set_expert(e, w13, w2)
            del w13, w2
        layer.set_router(wr, bias)
        return layer

    def sibling(self, bias: torch.Tensor | None = None, **shape_overrides) -> "MoeLayer":
        """A layer on the same device-resident weights with another routing
        configuration (e.g. n_groups, topk_groups) and bias; nothing is
        copied."""
        other = object.__new__(MoeLayer)
        other.shape = dict(self.shape, **shape_overrides)
        other.cfg = B.config_from(other.shape)
        other.E, other.device = self.E, self.device
        other.w13, other.s13, other.w2, other.s2, other.wr = self.w13, self.s13, self.w2, self.s2, self.wr
        other.bias = self.bias.clone() if bias is None else bias
        other.err = B.new_err_flag(self.device)
        other._ws = {}
        return other

    def weights(self) -> dict:
        return dict(w13=self.w13, s13=self.s13, w2=self.w2, s2=self.s2, wr=self.wr)

    # -------------------------------------------------------------- forward
    # Guard bands (bytes, a multiple of 256) around every workspace, filled
    # with GUARD_BYTE and checked by check_guards(): a kernel writing past
    # either end of its workspace shows up there.  Off (0) unless set.
    guard_bytes = 0
    GUARD_BYTE = 0xA5

    def workspace(self, T: int) -> torch.Tensor:
        ws = self._ws.get(T)
        if ws is None:
            n = max(B.moe_workspace_size(self.cfg, T), 256)
            g = self.guard_bytes
            if g:
                assert g % 256 == 0
                buf = torch.full((n + 2 * g,), self.GUARD_BYTE, dtype=torch.uint8, device=self.device)
                ws = buf[g:g + n]
                self._guarded = getattr(self, "_guarded", [])
                self._guarded.append((buf, g, n))
            else:
                ws = torch.empty(n, dtype=torch.uint8, device=self.device)
            self._ws[T] = ws
        return ws

    def check_guards(self) -> None:
        """Raise if any guard band around this layer's workspaces changed."""
        for buf, g, n in getattr(self, "_guarded", []):
            head, tail = buf[:g], buf[g + n:]
            if not (bool((head == self.GUARD_BYTE).all()) and bool((tail == self.GUARD_BYTE).all())):
                raise RuntimeError(f"workspace guard band overwritten (workspace of {n} bytes)")

    def forward(self, x: torch.Tensor, out=None, out_dtype=B.MOE_DTYPE_BF16, idx_out=None, counts_out=None,
                stream=None) -> torch.Tensor:
        return B.moe_forward(self.cfg, self.weights(), self.bias, x, out=out, out_dtype=out_dtype, idx_out=idx_out,
                             counts_out=counts_out, ws=self.workspace(x.shape[0]), err=self.err, stream=stream)

    def bias_update(self, counts: torch.Tensor, T: int, gamma: float = 0.001, stream=None) -> None:
        B.moe_bias_update(self.bias, counts, self.cfg.n_routed, T * self.cfg.top_k, gamma, stream=stream)

    def seq_balance_loss(self, T: int, seq_len: int, alpha: float = 1e-4, stream=None) -> torch.Tensor:
        """Sequence-wise balance loss of the batch of T tokens this layer's
        last forward of that size routed, one value per run of seq_len tokens."""
        return B.moe_seq_balance_loss(self.cfg, T, seq_len, self.workspace(T), self.err, alpha=alpha, stream=stream)

    def backward(self, x: torch.Tensor, dout: torch.Tensor, stream=None):
        """Gradients of the expert FFNs for the batch this layer's last forward
        of that size routed (routing held fixed): (dx, dW13, dW2) in FP32.
        The transposed weight copies the dgrad GEMMs read are made on first
        use (set-up) and kept."""
        if getattr(self, "_wt", None) is None:
            self._wt = B.moe_transpose_weights(self.cfg, self.weights(), stream=stream)
        T = x.shape[0]
        return B.moe_backward(self.cfg, self.weights(), self._wt, x, dout, self.workspace(T),
                              ws=self.backward_workspace(T), err=self.err, stream=stream)

    def backward_workspace(self, T: int) -> torch.Tensor:
        bws = getattr(self, "_bws", None)
        if bws is None:
            bws = self._bws = {}
        ws = bws.get(T)
        if ws is None:
            ws = torch.empty(max(int(B.lib.moe_backward_workspace_size(B.ctypes_cfg(self.cfg), T)), 256),
                             dtype=torch.uint8, device=self.device)
            bws[T] = ws
        return ws

    def check(self, stream=None) -> None:
        st, v = B.moe_check_device_error(self.err, stream)
        if st != B.MOE_OK:
            raise B.MoeError(st, f"device error flag {v:#x}")

    def layout(self, T: int) -> dict:
        return B.moe_workspace_layout(self.cfg, T)

"""Device-buffer plumbing for one MoE layer over the C ABI.

Nothing here computes: every step is one call into libexactmoe.so. torch is
used only to allocate device memory and to name the stream.
"""
from __future__ import annotations

import torch

from . import _native as N


class ExpertBank:
    """A device array of packed expert records (stride `rec` bytes).

    `pack` quantises BF16 expert weights on the device with moe_quantize_pack,
    writing codes and scales straight into the records.
    """

    def __init__(self, n_records: int, H: int, I: int, device="cuda"):
        self.H, self.I, self.n = H, I, n_records
        self.layout = N.moe_expert_record_layout(H, I)
        self.rec = self.layout["bytes"]
        self.buf = torch.empty(n_records * self.rec, dtype=torch.uint8, device=device)

    @property
    def ptr(self) -> int:
        return self.buf.data_ptr()

    def record_ptr(self, i: int) -> int:
        return self.ptr + i * self.rec

    def pack(self, gate, up, down, first: int = 0, stream=None):
        """gate, up [E][I][H], down [E][H][I] BF16 device tensors -> records first..first+E-1."""
        E = gate.shape[0]
        base = self.record_ptr(first)
        for w, q, s in ((gate, "gate_q", "gate_s"), (up, "up_q", "up_s"), (down, "down_q", "down_s")):
            w = w.contiguous()
            _, n, kk = w.shape
            N.moe_quantize_pack(w, E, n, kk, base + self.layout[q], self.rec, base + self.layout[s], self.rec, stream)

    def record_view(self, i: int) -> torch.Tensor:
        return self.buf[i * self.rec:(i + 1) * self.rec]

    def codes(self, i: int, part: str, rows: int, cols: int) -> torch.Tensor:
        """Packed codes of one matrix of record i as a [rows][cols/2] uint8 view."""
        off = i * self.rec + self.layout[part + "_q"]
        return self.buf[off:off + rows * cols // 2].view(rows, cols // 2)

    def scales(self, i: int, part: str, rows: int, cols: int) -> torch.Tensor:
        """BF16 scales of one matrix of record i as a [rows][cols/128] int16 view."""
        off = i * self.rec + self.layout[part + "_s"]
        return self.buf[off:off + rows * cols // 128 * 2].view(torch.int16).view(rows, cols // 128)


class Bf16Bank:
    """A device array of unquantised BF16 expert records (the BF16 baseline's
    weights): `load` copies gate, up [E][I][H] and down [E][H][I] BF16 tensors
    into the records at the offsets moe_bf16_record_layout gives."""

    def __init__(self, n_records: int, H: int, I: int, device="cuda"):
        self.H, self.I, self.n = H, I, n_records
        self.layout = N.moe_bf16_record_layout(H, I)
        self.rec = self.layout["bytes"]
        self.buf = torch.empty(n_records * self.rec, dtype=torch.uint8, device=device)

    @property
    def ptr(self) -> int:
        return self.buf.data_ptr()

    def load(self, gate, up, down, first: int = 0):
        E = gate.shape[0]
        recs = self.buf[first * self.rec:(first + E) * self.rec].view(E, self.rec)
        for w, part in ((gate, "gate"), (up, "up"), (down, "down")):
            n = w[0].numel() * 2
            off = self.layout[part]
            recs[:, off:off + n].copy_(w.contiguous().view(E, -1).view(torch.uint8))


# Up to this many tokens the router kernel also writes the FP16 copy of x
# that the grouped FFN multiplies (moe_route_topk_x16 + MOE_FFN_X_F16), so the
# FFN call runs no conversion pass; larger batches convert inside the FFN
# (gathered into group order for the tensor-core path).
ROUTER_X16_MAX_T = 64


class LayerBuffers:
    """Per-shape device buffers of one layer step (T tokens, top-k of E)."""

    def __init__(self, T: int, k: int, E: int, H: int, I: int, device="cuda", path=N.MOE_PATH_AUTO):
        self.T, self.k, self.E, self.H, self.I, self.path = T, k, E, H, I, path
        P = T * k
        d = dict(device=device)
        self.logits = torch.empty(max(T, 1), E, dtype=torch.bfloat16, **d)
        self.topk_ids = torch.empty(max(T, 1), k, dtype=torch.int32, **d)
        self.topk_w = torch.empty(max(T, 1), k, dtype=torch.float32, **d)
        self.counts = torch.empty(E, dtype=torch.int32, **d)
        self.offsets = torch.empty(E + 1, dtype=torch.int32, **d)
        self.sorted_pair = torch.empty(max(P, 1), dtype=torch.int32, **d)
        self.pair_pos = torch.empty(max(P, 1), dtype=torch.int32, **d)
        self.y = torch.empty(max(P, 1), H, dtype=torch.float32, **d)
        self.out = torch.empty(max(T, 1), H, dtype=torch.bfloat16, **d)
        self.group_ws_bytes = N.moe_group_workspace_size(T, k, E)
        self.group_ws = torch.zeros(self.group_ws_bytes, dtype=torch.uint8, **d)
        self.ffn_ws_bytes = N.moe_ffn_workspace_size(T, k, E, H, I, path)
        self.ffn_ws = torch.zeros(self.ffn_ws_bytes, dtype=torch.uint8, **d)
        self.x16 = torch.empty(T, H, dtype=torch.float16, **d) if 0 < T <= ROUTER_X16_MAX_T else None

    def ffn_input(self, x):
        """(activations, path) for moe_grouped_w4a16_ffn after this buffer's
        routing: the router's FP16 copy when it wrote one, else x itself."""
        return (self.x16, self.path | N.MOE_FFN_X_F16) if self.x16 is not None else (x, self.path)


def moe_layer_forward(x, w_router, bank: ExpertBank, buf: LayerBuffers, *, bias=None, flags=0,
                      expert_slot=None, n_slots=None, residual=None, out=None, stream=None):
    """route -> group -> grouped FFN -> combine for x [T][H]; returns `out`."""
    T, k, E, H, I = buf.T, buf.k, buf.E, buf.H, buf.I
    out = buf.out if out is None else out
    if buf.x16 is not None:  # the router also writes the FFN's FP16 input; range errors go to the FFN's word
        N.moe_route_topk_x16(x, w_router, T, H, E, k, bias, flags, buf.logits, buf.topk_ids, buf.topk_w,
                             buf.x16, buf.ffn_ws, stream)
    else:
        N.moe_route_topk(x, w_router, T, H, E, k, bias, flags, buf.logits, buf.topk_ids, buf.topk_w, stream)
    N.moe_group_tokens(buf.topk_ids, T, k, E, buf.counts, buf.offsets, buf.sorted_pair, buf.pair_pos,
                       buf.group_ws, buf.group_ws_bytes, stream)
    x_ffn, path = buf.ffn_input(x)
    N.moe_grouped_w4a16_ffn(x_ffn, buf.sorted_pair, buf.offsets, bank.ptr, bank.rec, expert_slot,
                            bank.n if n_slots is None else n_slots, T, k, E, H, I, path, buf.y,
                            buf.ffn_ws, buf.ffn_ws_bytes, stream)
    N.moe_combine(buf.y, buf.topk_w, buf.pair_pos, residual, T, k, H, out, stream)
    return out

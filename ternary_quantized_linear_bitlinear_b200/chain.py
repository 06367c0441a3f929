"""A dependency-ordered decode step through a stack of BitLinear layers.

Each layer feeds the next, as one token step of a decoder does, with every
projection a BitLinear of this library and nothing computed outside it:

    Y_q, Y_k, Y_v = BitLinear_{q,k,v}(x)           one fused decode launch
    Y_o           = BitLinear_o(SubLN(Y_q))        one fused decode launch
    Y_g, Y_u      = BitLinear_{gate,up}(Y_o)       one fused decode launch
    x_q, s        = quant(SubLN(relu(Y_g)^2 Y_u))  bl_ffn_act_quant
    x'            = BitLinear_down(x_q, s)         one decode launch
    (x' is the next layer's x)

Attention is outside this library, so the o projection reads the q
projection's output in its place (same width); SubLN sits before o_proj and
down_proj ("BitDistill", Stage 1 -- Architectural refinement with SubLN),
ReLU^2 gates the FFN ("SLM750-Edge", Key Architectural Features).  The
weights are static, so every projection launch is a programmatic dependent
of the launch before it (BL_FWD_WEIGHTS_READY): it streams its weights while
that launch finishes, and reads its activations only after.

This module only arranges buffers and calls the library's entry points.
"""
from __future__ import annotations

import torch

from . import api

# projection order inside a layer, and the launch groups of one layer
PROJ = ("q", "k", "v", "o", "gate", "up", "down")


class DecodeChain:
    """layers: list of dicts name -> (packed uint8 [N, K/4], gamma float32 [1],
    N, K) for the seven projections; gains: list of (g_o [hidden],
    g_down [ffn]) float32 device tensors.  M tokens per step (M <= 16).
    With record=True every projection also writes its x_q, s and int32
    accumulators (for checking), else only Y."""

    def __init__(self, layers, gains, M: int, eps: float = 1e-6, record: bool = False):
        self.M = M
        self.eps = eps
        self.record = record
        self.L = api.lib()
        dev = layers[0]["q"][0].device
        hidden = layers[0]["q"][3]
        ffn = layers[0]["gate"][2]
        self.x0 = torch.zeros(M, hidden, dtype=torch.float32, device=dev)
        self.layers = []
        x_in = self.x0
        for li, (lay, (g_o, g_d)) in enumerate(zip(layers, gains)):
            bufs = {}
            for name in PROJ:
                packed, gamma, N, K = lay[name]
                b = dict(packed=packed, gamma=gamma, N=N, K=K,
                         Y=torch.empty(M, N, dtype=torch.float32, device=dev))
                if record:
                    b["x_q"] = torch.empty(M, K, dtype=torch.int8, device=dev)
                    b["s"] = torch.empty(max(M, 4), dtype=torch.float32, device=dev)[:M]
                    b["acc"] = torch.empty(M, N, dtype=torch.int32, device=dev)
                bufs[name] = b
            bufs["ffn_xq"] = torch.empty(M, ffn, dtype=torch.int8, device=dev)
            bufs["ffn_s"] = torch.empty(max(M, 4), dtype=torch.float32, device=dev)[:M]
            bufs["x_in"] = x_in
            bufs["g_o"], bufs["g_d"] = g_o, g_d

            def dec(names, X, gain):
                items = []
                for n in names:
                    b = bufs[n]
                    items.append((b["packed"], b["gamma"], X, gain, b["Y"], b.get("x_q"), b.get("s"), b.get("acc"),
                                  b["N"], b["K"]))
                return api.make_decode_problems(items, M=M), len(items)

            d = bufs["down"]
            bufs["launch_qkv"] = dec(("q", "k", "v"), x_in, None)
            bufs["launch_o"] = dec(("o",), bufs["q"]["Y"], g_o)
            bufs["launch_gu"] = dec(("gate", "up"), bufs["o"]["Y"], None)
            bufs["launch_down"] = (api.make_problems([(d["packed"], d["gamma"], bufs["ffn_xq"], bufs["ffn_s"], d["Y"],
                                                       d.get("acc"), d["N"], d["K"])], M=M), 1)
            self.layers.append(bufs)
            x_in = d["Y"]
        self.out = x_in

    def launches_per_step(self) -> int:
        return 5 * len(self.layers)

    def run(self, stream_ptr: int):
        """Enqueue one token step on the raw stream handle (graph-capturable)."""
        L, M, eps = self.L, self.M, self.eps
        RDY = api.BL_FWD_WEIGHTS_READY
        for b in self.layers:
            for key in ("launch_qkv", "launch_o", "launch_gu"):
                arr, n = b[key]
                rc = L.bl_linear_decode_grouped(arr, n, api.BL_F32, M, eps, RDY, stream_ptr)
                if rc:
                    raise api.BitLinearError(rc, "bl_linear_decode_grouped")
            g, u = b["gate"]["Y"], b["up"]["Y"]
            rc = L.bl_ffn_act_quant(g.data_ptr(), u.data_ptr(), M, g.shape[1], b["g_d"].data_ptr(), eps,
                                    b["ffn_xq"].data_ptr(), b["ffn_s"].data_ptr(), stream_ptr)
            if rc:
                raise api.BitLinearError(rc, "bl_ffn_act_quant")
            arr, n = b["launch_down"]
            rc = L.bl_forward_grouped(arr, n, M, RDY, stream_ptr)
            if rc:
                raise api.BitLinearError(rc, "bl_forward_grouped")

"""The MoE layer forward as a fixed sequence of libmoe calls.

"MoE 混合专家模型推理参数与前向传播详解" §3 gives the order: routing (§3.1),
permutation (§3.2), routed experts as one grouped GEMM and the shared experts
(§3.3), unpermute + combine (§3.4). Between forwards the xxqk.cn digest §2.2
adds the aux-loss-free bias step. torch only provides the device buffers and
the stream; there is no host synchronisation inside a forward.
"""
from dataclasses import dataclass
from typing import Optional

import torch

from . import native as N


@dataclass
class LayerSpec:
    H: int
    E: int
    I: int
    I_s: int
    k: int
    n_group: int
    topk_group: int
    scoring: str             # "softmax" | "sigmoid"
    norm_topk_prob: bool
    scale: float
    dtype: str = "bf16"      # expert weights / activations: "bf16" | "e4m3"

    @classmethod
    def from_config(cls, cfg):
        return cls(cfg.H, cfg.E, cfg.I, cfg.I_s, cfg.k, cfg.n_group, cfg.topk_group,
                   cfg.scoring, cfg.norm_topk_prob, cfg.scale, cfg.dtype)


class MoELayer:
    """Holds the weights (device tensors) and the per-forward buffers."""

    def __init__(self, spec: LayerSpec, gate: torch.Tensor, w13: torch.Tensor, w2: torch.Tensor,
                 sw13: Optional[torch.Tensor], sw2: Optional[torch.Tensor],
                 bias: Optional[torch.Tensor], T_max: int, gather: bool = False,
                 fuse_shared: bool = True, fuse_combine: bool = False, fuse_ffn: Optional[bool] = None,
                 tiled_weights: bool = True):
        self.spec = spec
        # gather=True: bf16 layers read the routed experts' token rows straight
        # from x (the permutation fused into the first GEMM; no x_perm). At the
        # V3 shape on B200 the TMA path over x_perm is faster, so it is off.
        self.gather = gather and spec.dtype != "e4m3"
        # fuse_shared: the shared expert's GEMMs share the routed experts' launches
        self.fuse_shared = fuse_shared
        # fuse_combine: the combine runs inside the down GEMM (atomic fp32 adds
        # into a [T, H] accumulator); measured slower at the V3 shape, so off
        self.fuse_combine = fuse_combine and spec.dtype != "e4m3"
        # fuse_ffn: bf16 layers with a shared expert run both GEMMs (routed and
        # shared) as one persistent launch on a dynamic tile counter, down
        # tiles starting as soon as their token block's h rows are stored.
        # None: by shape, per forward: when the routed rows average at least
        # two full 256-row token blocks per expert (measured on B200: 11 %
        # faster at 1024 rows per expert, level at 256 and 384)
        self.fuse_ffn = fuse_ffn
        self.ffn_ok = (fuse_ffn is not False and spec.dtype != "e4m3" and fuse_shared and not self.gather
                       and not self.fuse_combine and spec.I_s > 0 and sw13 is not None)
        dev = gate.device
        self.dev = dev
        self.gate = gate.contiguous()
        self.bias = bias.contiguous().clone() if bias is not None else None
        self.fp8 = spec.dtype == "e4m3"
        H, E, I, I_s, k = spec.H, spec.E, spec.I, spec.I_s, spec.k
        if self.fp8:
            # E4M3 weights with 128x128 block scales, quantised once by libmoe
            self.w13, self.w13_s = self._quant_blocks(w13)
            self.w2, self.w2_s = self._quant_blocks(w2)
            if sw13 is not None:
                self.sw13, self.sw13_s = self._quant_blocks(sw13.unsqueeze(0))
                self.sw2, self.sw2_s = self._quant_blocks(sw2.unsqueeze(0))
            else:
                self.sw13 = self.sw2 = self.sw13_s = self.sw2_s = None
        else:
            self.w13, self.w2 = w13.contiguous(), w2.contiguous()
            self.w13_s = self.w2_s = None
            self.sw13 = sw13.contiguous() if sw13 is not None else None
            self.sw2 = sw2.contiguous() if sw2 is not None else None
            self.sw13_s = self.sw2_s = None
            if tiled_weights:
                # the layer's own copies in the tiled layout (each weight tile
                # the GEMMs load in one step is contiguous in HBM; 3 % faster
                # GEMMs at the V3 shape on B200). They are new tensors of the
                # weights' size: the caller may free its row-major ones.
                # tiled_weights=False reads the caller's tensors as they are.
                self.w13, self.w2 = self._tiled(self.w13, self.w2, E, I)
                if self.sw13 is not None:
                    self.sw13, self.sw2 = self._tiled(self.sw13, self.sw2, 1, I_s)
        # bf16 weights held tiled (moe_tile_ffn_weights); E4M3 ones row-major
        self.tiled = tiled_weights and not self.fp8
        self.T_max = T_max
        R = T_max * k
        i32, f32, bf = torch.int32, torch.float32, torch.bfloat16
        act = torch.uint8 if self.fp8 else bf
        z = lambda *s, dt: torch.empty(*s, dtype=dt, device=dev)
        self.logits = z(T_max, E, dt=f32)
        self.ids = z(T_max, k, dt=i32)
        self.topk_w = z(T_max, k, dt=f32)
        self.counts = z(E, dt=i32)
        self.offsets = z(E + 1, dt=i32)
        self.src_token = z(R, dt=i32)
        self.slot_to_row = z(R, dt=i32)
        self.row_w = z(R, dt=f32)
        ws = N.moe_permute_workspace_size(T_max, k, E)
        self.ws = z((ws + 15) // 16 * 16, dt=torch.uint8)
        self.x_perm = None if self.gather else z(R, H, dt=act)
        self.h = z(R, I, dt=act)
        self.o = z(R, H, dt=bf)
        self.y = z(T_max, H, dt=bf)
        self.load_cv = z(1, dt=f32)
        self.y_acc = z(T_max, H, dt=f32) if self.fuse_combine else None
        self.status = torch.zeros(1, dtype=i32, device=dev)
        if self.fp8:
            self.xq = z(T_max, H, dt=torch.uint8)
            self.xs = z(T_max, H // 128, dt=f32)
            self.x_perm_s = z(R, H // 128, dt=f32)
            self.h_s = z(R, I // 128, dt=f32)
            self.sh_h_s = z(T_max, max(I_s, 128) // 128, dt=f32)
        else:
            self.xq = self.xs = self.x_perm_s = self.h_s = self.sh_h_s = None
        if I_s > 0:
            self.sh_h = z(T_max, I_s, dt=act)
            self.sh_o = z(T_max, H, dt=bf)
        else:
            self.sh_h = self.sh_o = None
        if self.ffn_ok:
            n = N.moe_swiglu_ffn_sync_size(R, E, T_max)
            self.ffn_ws = z((n + 15) // 16 * 16, dt=torch.uint8)
        else:
            self.ffn_ws = None

    def _tiled(self, w13, w2, groups, I):
        t13, t2 = torch.empty_like(w13), torch.empty_like(w2)
        N.moe_tile_ffn_weights(self.spec.H, w13, w2, groups, I, t13, t2)
        return t13, t2

    def _quant_blocks(self, w):
        B, Nr, K = w.shape
        q = torch.empty(B, Nr, K, dtype=torch.uint8, device=w.device)
        s = torch.empty(B, Nr // 128, K // 128, dtype=torch.float32, device=w.device)
        N.moe_quantize_blocks(B, Nr, K, w.contiguous(), q, s)
        return q, s

    # -------------------------------------------------------------- stages
    def route(self, x: torch.Tensor, write_logits: bool = False, logits_in: Optional[torch.Tensor] = None):
        s = self.spec
        T = (logits_in if logits_in is not None else x).shape[0]
        N.moe_route(T, s.H, s.E, s.k, s.n_group, s.topk_group,
                    N.MOE_SIGMOID if s.scoring == "sigmoid" else N.MOE_SOFTMAX,
                    s.norm_topk_prob, s.scale,
                    None if logits_in is not None else x,
                    self.gate, self.bias,
                    logits_in if logits_in is not None else self.logits[:T],
                    self.ids[:T], self.topk_w[:T], self.counts, self.status)

    def permute(self, x: torch.Tensor, T: int):
        """The permutation; E4M3 layers quantise x per 1x128 tile inside it
        (x_perm codes + scales, and the unpermuted codes xq / xs the shared
        expert reads)."""
        s = self.spec
        R = T * s.k
        if self.fp8:
            N.moe_permute(T, s.k, s.E, s.H, self.ids[:T], self.topk_w[:T], x, N.MOE_BF16, None,
                          self.x_perm[:R], self.x_perm_s[:R], self.offsets, self.src_token[:R],
                          self.slot_to_row[:R], self.row_w[:R], self.ws, self.status,
                          perm_dtype=N.MOE_E4M3, x_q=self.xq[:T] if self.sh_h is not None else None,
                          x_q_scale=self.xs[:T] if self.sh_h is not None else None)
            return
        N.moe_permute(T, s.k, s.E, s.H, self.ids[:T], self.topk_w[:T], x, N.MOE_BF16, None,
                      None if self.gather else self.x_perm[:R], None,
                      self.offsets, self.src_token[:R], self.slot_to_row[:R], self.row_w[:R],
                      self.ws, self.status)

    def _dt(self):
        return N.MOE_E4M3 if self.fp8 else N.MOE_BF16

    def experts_gate_up(self, T: int, x: Optional[torch.Tensor] = None):
        s = self.spec
        R = T * s.k
        if self.gather:
            N.moe_gate_up_swiglu_gather(R, s.H, self.w13, s.E, s.I, x, T, self.src_token[:R],
                                        self.offsets, self.h[:R], dev_status=self.status,
                                        tiled=self.tiled)
            return
        N.moe_gate_up_swiglu(R, s.H, self.w13, self._dt(), s.E, s.I, self.x_perm[:R], self.offsets,
                             self.h[:R], w13_scale=self.w13_s,
                             a_scale=self.x_perm_s[:R] if self.fp8 else None,
                             h_scale_ws=self.h_s[:R] if self.fp8 else None, dev_status=self.status,
                             tiled=self.tiled)

    def experts_down(self, T: int):
        s = self.spec
        R = T * s.k
        N.moe_down_proj(R, s.H, self.w2, self._dt(), s.E, s.I, self.h[:R], self.offsets,
                        self.row_w[:R], self.o[:R], w2_scale=self.w2_s,
                        h_scale=self.h_s[:R] if self.fp8 else None, dev_status=self.status,
                        tiled=self.tiled)

    def shared_gate_up(self, x: torch.Tensor, T: int):
        s = self.spec
        a = self.xq[:T] if self.fp8 else x
        N.moe_gate_up_swiglu(T, s.H, self.sw13, self._dt(), 1, s.I_s, a, None, self.sh_h[:T],
                             w13_scale=self.sw13_s, a_scale=self.xs[:T] if self.fp8 else None,
                             h_scale_ws=self.sh_h_s[:T] if self.fp8 else None,
                             dev_status=self.status, tiled=self.tiled)

    def shared_down(self, T: int):
        s = self.spec
        N.moe_down_proj(T, s.H, self.sw2, self._dt(), 1, s.I_s, self.sh_h[:T], None, None,
                        self.sh_o[:T], w2_scale=self.sw2_s,
                        h_scale=self.sh_h_s[:T] if self.fp8 else None, dev_status=self.status,
                        tiled=self.tiled)

    def gate_up_with_shared(self, x: torch.Tensor, T: int):
        """Routed experts' and shared expert's first GEMM in one launch."""
        s = self.spec
        R = T * s.k
        N.moe_gate_up_swiglu_with_shared(
            R, s.H, self.w13, self._dt(), s.E, s.I, self.x_perm[:R], self.offsets, self.h[:R],
            T, self.sw13, s.I_s, self.xq[:T] if self.fp8 else x, self.sh_h[:T],
            w13_scale=self.w13_s, a_scale=self.x_perm_s[:R] if self.fp8 else None,
            h_scale_ws=self.h_s[:R] if self.fp8 else None, sw13_scale=self.sw13_s,
            sh_a_scale=self.xs[:T] if self.fp8 else None,
            sh_h_scale_ws=self.sh_h_s[:T] if self.fp8 else None, dev_status=self.status,
            tiled=self.tiled)

    def down_with_shared(self, T: int):
        """Routed experts' and shared expert's second GEMM in one launch."""
        s = self.spec
        R = T * s.k
        N.moe_down_proj_with_shared(
            R, s.H, self.w2, self._dt(), s.E, s.I, self.h[:R], self.offsets, self.row_w[:R], self.o[:R],
            T, self.sw2, s.I_s, self.sh_h[:T], self.sh_o[:T], w2_scale=self.w2_s,
            h_scale=self.h_s[:R] if self.fp8 else None, sw2_scale=self.sw2_s,
            sh_h_scale=self.sh_h_s[:T] if self.fp8 else None, dev_status=self.status,
            tiled=self.tiled)

    def ffn_with_shared(self, x: torch.Tensor, T: int):
        """Both GEMMs of the routed experts and of the shared expert in one launch."""
        s = self.spec
        R = T * s.k
        N.moe_swiglu_ffn_with_shared(
            R, s.H, self.w13, self.w2, s.E, s.I, self.x_perm[:R], self.offsets, self.row_w[:R], self.h[:R],
            self.o[:R], T, self.sw13, self.sw2, s.I_s, x, self.sh_h[:T], self.sh_o[:T], self.ffn_ws,
            dev_status=self.status, tiled=self.tiled)

    def down_with_combine(self, T: int):
        """The routed and shared down GEMMs with the combine in their epilogue."""
        s = self.spec
        R = T * s.k
        N.moe_down_proj_combine(R, T, s.H, self.w2, s.E, s.I, self.h[:R], self.offsets, self.row_w[:R],
                                self.src_token[:R], self.sw2, s.I_s,
                                self.sh_h[:T] if self.sh_h is not None else None,
                                self.y_acc[:T], self.y[:T], dev_status=self.status,
                                tiled=self.tiled)

    def combine(self, T: int):
        s = self.spec
        N.moe_combine(T, s.k, s.H, self.o[:T * s.k], self.slot_to_row[:T * s.k], None,
                      self.sh_o[:T] if self.sh_o is not None else None, self.y[:T])

    def stages(self, x: torch.Tensor, write_logits: bool = False):
        """The forward as named steps, each one or more libmoe launches."""
        T = x.shape[0]
        assert T <= self.T_max and x.dtype == torch.bfloat16 and x.is_contiguous()
        st = [("route", lambda: self.route(x, write_logits)),
              ("permute", lambda: self.permute(x, T))]
        if self.fuse_combine:
            if self.sh_h is not None and not self.gather:
                st.append(("gate_up", lambda: self.gate_up_with_shared(x, T)))
            else:
                st.append(("gate_up_routed", lambda: self.experts_gate_up(T, x)))
                if self.sh_h is not None:
                    st.append(("gate_up_shared", lambda: self.shared_gate_up(x, T)))
            st.append(("down_combine", lambda: self.down_with_combine(T)))
            return st
        if self.ffn_ok and (self.fuse_ffn or T * self.spec.k >= 512 * self.spec.E):
            # routed + shared expert, both GEMMs, one launch
            st.append(("ffn", lambda: self.ffn_with_shared(x, T)))
        elif self.sh_h is not None and self.fuse_shared and not self.gather:
            # routed + shared expert in one launch per GEMM
            st += [("gate_up", lambda: self.gate_up_with_shared(x, T)),
                   ("down", lambda: self.down_with_shared(T))]
        else:
            st += [("gate_up_routed", lambda: self.experts_gate_up(T, x)),
                   ("down_routed", lambda: self.experts_down(T))]
            if self.sh_h is not None:
                st += [("gate_up_shared", lambda: self.shared_gate_up(x, T)),
                       ("down_shared", lambda: self.shared_down(T))]
        st.append(("combine", lambda: self.combine(T)))
        return st

    def forward(self, x: torch.Tensor, write_logits: bool = False) -> torch.Tensor:
        """y = shared(x) + sum_j w_j E_j(x) for the T rows of x (bf16 [T, H])."""
        for _, run in self.stages(x, write_logits):
            run()
        return self.y[:x.shape[0]]

    def capture(self, x: torch.Tensor, bias_gamma: Optional[float] = None):
        """Records the forward on the rows of x (and, with bias_gamma, the
        bias step after it) as one CUDA graph; returns the function that
        replays it on the current stream. The graph keeps x's and the layer's
        buffers: refill x in place between replays. Every launch of the
        forward is one node, so a replay costs one launch on the host."""
        T = x.shape[0]
        stages = self.stages(x)
        side = torch.cuda.Stream(device=self.dev)
        side.wait_stream(torch.cuda.current_stream(self.dev))
        with torch.cuda.stream(side):                   # first run outside the capture
            for _, run in stages:
                run()
        torch.cuda.current_stream(self.dev).wait_stream(side)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for _, run in stages:
                run()
            if bias_gamma is not None:
                self.bias_step(T, bias_gamma, load_cv=False)
        self._graphs = getattr(self, "_graphs", []) + [graph]   # kept alive with the layer
        return graph.replay

    def bias_step(self, T: int, gamma: float, load_cv: bool = True):
        """Aux-loss-free bias update from the last forward's expert counts."""
        s = self.spec
        if self.bias is None:
            raise ValueError("layer has no selection bias")
        N.moe_bias_update(s.E, T, s.k, self.counts, self.bias, gamma,
                          self.load_cv if load_cv else None)

    def aux_loss(self, T: int, seq_len: Optional[int] = None, alpha: float = 0.001) -> torch.Tensor:
        """Sequence-level auxiliary balance loss of the last forward ("MoE 混合
        专家模型推理参数与前向传播详解" §6.2), from its logits and expert ids;
        a [1] fp32 device tensor, alpha * mean over sequences of seq_len
        tokens (default: the T tokens as one sequence)."""
        s = self.spec
        seq_len = T if seq_len is None else seq_len
        ws = torch.empty(N.moe_aux_loss_workspace_size(T, s.E, seq_len), dtype=torch.uint8, device=self.dev)
        out = torch.empty(1, dtype=torch.float32, device=self.dev)
        N.moe_aux_loss(T, s.E, s.k, seq_len, N.MOE_SIGMOID if s.scoring == "sigmoid" else N.MOE_SOFTMAX,
                       self.logits[:T], self.ids[:T], alpha, out, ws, self.status)
        return out

    def device_status(self) -> int:
        return N.moe_read_device_status(self.status)

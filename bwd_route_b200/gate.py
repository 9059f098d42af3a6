"""One full pass of the top-1 MoE gate through the C ABI.

MoETop1Gate owns the device buffers (allocated with torch: plumbing only) and
runs, in stream order, the five library calls of a training step:

    moe_top1_route -> moe_top1_fwd -> moe_top1_bwd -> moe_aux_loss_fwd_bwd
    -> moe_lambda_eff_update

The step mirrors the training loop of foxhunt commit 9170d24fe3 ("Single
source of truth for the attention path", PerceptionTrainer integration):
forward through the MoE dispatch, backward through it, then the load-balance
loss, whose weight lambda_eff is read from device memory and updated by the
controller of foxhunt commit 2d0e6b6bdc at the end of the step.

Beside step(): forward_mean_collapse / backward_mean_collapse when the gate's
output is averaged over the horizon axis (ctx_mean [B, H]); update_controller,
which produces ent_ema from the step's expert usage and recomputes lambda_eff;
and, for data-parallel jobs, enable_data_parallel / allreduce_gradients.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import dp, ops


class MoETop1Gate:
    # kernels launched per step with T > 0: route 2 (count; scatter with the
    # scan folded in) while ceil(T / 1024) * E <= 32768, else 3 (a separate scan);
    # fwd 1; bwd 3 (d_x, the weight-gradient contraction and the slot reduction),
    # or 2 where the TF32 backward takes one fused pass for both contractions
    # (the horizon-mean gradient at H = 256; H = 128 above 65,536 tokens), then the
    # reduction; aux with the lambda update 1 (its
    # last block finalizes the loss, then writes the next lambda)
    @staticmethod
    def launches_per_step(math: int, H: int, T: int, E: int, mean_collapse: bool = False) -> int:
        route = 2 if -(-T // 1024) * E <= 32768 else 3
        single = math == ops.MOE_MATH_TF32 and ((mean_collapse and H == 256) or (H == 128 and T > 65536))
        bwd = 2 if single else 3
        return route + 1 + bwd + 1  # aux and the lambda update share one launch

    def __init__(self, W: torch.Tensor, bias: torch.Tensor, B: int, N_H: int, math: int = ops.MOE_MATH_TF32,
                 lambda_floor: float = 0.01, lambda_max_extra: float = 0.09, ent_target: float = 1.0,
                 ent_ema: float = 0.0, stats: bool = True):
        assert W.is_cuda and W.dtype == torch.float32 and W.dim() == 3
        self.E, self.H = W.shape[0], W.shape[1]
        self.B, self.N_H, self.T = B, N_H, B * N_H
        self.math = math
        self.W, self.bias = W, bias
        dev = W.device
        f32 = torch.float32
        T, E, H = self.T, self.E, self.H
        self.lambda_floor, self.lambda_max_extra, self.ent_target = lambda_floor, lambda_max_extra, ent_target
        self.routing = ops.Routing.empty(T, E, dev)
        self.routed = torch.empty(T, H, dtype=f32, device=dev)
        self.d_x = torch.empty(T, H, dtype=f32, device=dev)
        self.ctx_mean = torch.empty(B, H, dtype=f32, device=dev)
        # dW and db are views of one flat buffer, so that a data-parallel step sums
        # both over the ranks with one collective (db starts E*H*H*4 bytes in: a
        # multiple of 4 KiB for every supported H)
        self.grads = torch.empty(E * H * H + E * H, dtype=f32, device=dev)
        self.dW = self.grads[:E * H * H].view(E, H, H)
        self.db = self.grads[E * H * H:].view(E, H)
        self.d_logits = torch.empty(T, E, dtype=f32, device=dev)
        self.loss = torch.zeros(2, dtype=f32, device=dev)
        self.mean_p = torch.zeros(E, dtype=f32, device=dev)
        self.stats = torch.zeros(3 * E + 4, dtype=f32, device=dev) if stats else None
        self.lambda_eff = torch.full((1,), lambda_floor, dtype=f32, device=dev)
        self.ent_ema = torch.full((1,), ent_ema, dtype=f32, device=dev)
        self.usage_ema = torch.full((E,), 1.0 / E, dtype=f32, device=dev)
        self.ent_step = torch.zeros(1, dtype=f32, device=dev)
        self.ws = ops.new_workspace(T, E, H, dev)
        self.dp_group = None
        self.dp_tokens = T
        self.counts_global = None

    def route(self, gate_logits, stream=None):
        ops.moe_top1_route(gate_logits, self.B, self.N_H, self.E, self.routing, self.ws, stream)

    def forward(self, x, stream=None):
        ops.moe_top1_fwd(x, self.W, self.bias, self.routing, self.B, self.N_H, self.E, self.H, self.math,
                         self.routed, self.ws, stream)

    def forward_mean_collapse(self, x, stream=None):
        """Forward followed by the horizon mean: ctx_mean [B, H] (no [T, H] output)."""
        ops.moe_top1_fwd_mean_collapse(x, self.W, self.bias, self.routing, self.B, self.N_H, self.E, self.H, self.math,
                                       self.ctx_mean, self.ws, stream)

    def backward(self, x, d_out, stream=None):
        ops.moe_top1_bwd(x, self.W, d_out, self.routing, self.B, self.N_H, self.E, self.H, self.math, self.d_x,
                         self.dW, self.db, 0, self.ws, stream)

    def backward_mean_collapse(self, x, grad_ctx_mean, stream=None):
        """Backward when the gate's output is averaged over the horizon axis:
        grad_ctx_mean [B, H] is the gradient of that mean."""
        ops.moe_top1_bwd_mean_collapse(x, self.W, grad_ctx_mean, self.routing, self.B, self.N_H, self.E, self.H,
                                       self.math, self.d_x, self.dW, self.db, 0, self.ws, stream)

    def aux(self, gate_logits, stream=None):
        ops.moe_aux_loss_fwd_bwd(gate_logits, self.routing.counts, self.B, self.N_H, self.E, self.lambda_eff,
                                 self.d_logits, self.loss, self.mean_p, self.stats, self.ws, stream)

    def aux_and_update_lambda(self, gate_logits, stream=None):
        """aux() and then update_lambda() in one launch (the same bits)."""
        ops.moe_aux_loss_fwd_bwd_lambda_update(gate_logits, self.routing.counts, self.B, self.N_H, self.E,
                                               self.lambda_eff, self.d_logits, self.loss, self.mean_p, self.stats,
                                               self.ent_ema, self.lambda_floor, self.lambda_max_extra,
                                               self.ent_target, self.lambda_eff, self.ws, stream)

    def update_lambda(self, stream=None):
        ops.moe_lambda_eff_update(self.ent_ema, self.lambda_floor, self.lambda_max_extra, self.ent_target,
                                  self.lambda_eff, stream)

    def update_controller(self, alpha: float, reset: bool = False, stream=None):
        """Closes the lambda loop after a step: the gate-entropy producer folds
        this step's usage into ent_ema (or resets it at a fold boundary), then
        lambda_eff is recomputed from it for the next step. Under data
        parallelism the usage is that of the global batch (counts summed over
        the ranks), so every rank holds the same ent_ema and lambda_eff."""
        counts = self.routing.counts
        if self.dp_group is not None:
            self._dp_stream_check(stream)
            counts = dp.global_counts(counts, self.counts_global, self.dp_group)
        ops.moe_usage_entropy_ema_update(counts, self.dp_tokens, self.E, alpha, reset, self.usage_ema,
                                         self.ent_ema, self.ent_step, stream)
        self.update_lambda(stream)

    def enable_data_parallel(self, group=None):
        """Makes this gate one replica of a data-parallel job over the ranks of
        group (torch.distributed, initialised by the caller; NCCL on GPUs).
        Every rank must hold a shard of the same [B, N_H] shape."""
        self.dp_tokens = dp.world_tokens(self.T, self.W.device, group)
        self.counts_global = torch.zeros(self.E, dtype=torch.int32, device=self.W.device)
        self.dp_group = group if group is not None else dist.group.WORLD

    def allreduce_gradients(self, stream=None):
        """After backward: dW and db of the global batch on every rank (their
        sum over the ranks' shards). A no-op without data parallelism."""
        if self.dp_group is None:
            return
        self._dp_stream_check(stream)
        dp.allreduce_gradients(self.grads, self.dp_group)

    @staticmethod
    def _dp_stream_check(stream):
        if stream is not None and stream != torch.cuda.current_stream():
            raise ValueError("a data-parallel step runs on torch's current stream")

    def step(self, gate_logits, x, d_out, stream=None):
        self.route(gate_logits, stream)
        self.forward(x, stream)
        self.backward(x, d_out, stream)
        self.aux_and_update_lambda(gate_logits, stream)

"""CPU oracle for the fused MoE expert layer -- TEST INFRASTRUCTURE ONLY.

This package is the plain, slow, obviously-correct definition of what the CUDA library
computes.  Only the test-suite, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import it; the library itself never does, and this package never imports the
library.  The two share no code: the oracle has its own number-format codecs, its own fp32
exponential and its own routing, dispatch, FFN and combine, all written from the source
pages' statement of the method:

* jiqizhixin, "DeepSeek悄悄更新：Mega MoE、FP4 Indexer来了", section "Mega MoE 是什么？":
  a conventional MoE layer runs dispatch -> linear -> SwiGLU -> linear -> combine as separate
  steps; Mega MoE fuses dispatch, both linears, SwiGLU and combine into one kernel; FP8 x FP4
  mixed precision.
* youleyou, "DeepSeek 模型更新解读 Tile Kernels 与 DeepEP V2 新特性", section
  "Tile Kernels：逼近硬件极限的底层优化", feature list: gating = top-k expert selection with
  scoring; MoE routing = token-to-expert mapping with fused expand / reduce and weight
  normalisation; quantisation = FP8/FP4 per-token / per-block, fused with SwiGLU.

The pages fix the steps and their order, not the formulas.  Where they are silent the oracle
takes one plain reading, stated in the function that implements it:

* router: softmax (select on raw logits, gates = softmax over the k selected, i.e. the
  renormalised top-k of the full softmax) or sigmoid + per-expert selection bias
  (select on sigmoid(l) + b, gates = sigmoid(l) renormalised over the selected);
  ties go to the lower expert id; the sigmoid keys are evaluated in fp32 with the
  project's own exponential so that both implementations take the selection decision on
  identical fp32 keys;
* dispatch: stable counting sort, slots of one expert in ascending token order;
* W1 rows [0, I) are the gate projection and rows [I, 2I) the up projection;
* h = silu(gate) * up is stored in the activation format (fp32 / BF16 / E4M3 with one
  power-of-two scale per 1x128 block, the smallest 2^n with amax <= 448 * 2^n); y and the
  output are BF16 (fp32 for the fp32 layer); the combine sums the k expert outputs in rank
  order.

``oracle.backward`` (imported by name, not re-exported here) holds the gradients of the
same layer's fp64 definition, pinned by finite differences and torch autograd.

Every function accumulates in fp64 and applies each storage rounding of the layer's data
contract at the point where the CUDA path stores that tensor.
"""
from .formats import (e4m3_decode, e4m3_encode, e2m1_decode_packed, ue8m0_decode,
                      bf16_bits_to_f64, round_bf16, round_bf16_bits)
from .fexp import exp_f32, sigmoid_f32
from .moe import (route, dispatch, dequant_x, dequant_w, quant_e4m3_1x128, expert_ffn,
                  combine, forward, forward_tokens, ffn_slots, Layer, quantize_activations)

__all__ = [
    "e4m3_decode", "e4m3_encode", "e2m1_decode_packed", "ue8m0_decode", "bf16_bits_to_f64",
    "round_bf16", "round_bf16_bits", "exp_f32", "sigmoid_f32", "route", "dispatch",
    "dequant_x", "dequant_w", "quant_e4m3_1x128", "expert_ffn", "combine", "forward",
    "forward_tokens", "ffn_slots", "Layer", "quantize_activations",
]

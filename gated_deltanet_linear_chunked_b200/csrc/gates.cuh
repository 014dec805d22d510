// gates.cuh -- the gate activations of the fused GDN prologue.
//
// A GDN block's gate layer emits two logits per (token, head): x for the
// decay and y for the write strength.  The pages name the gate layer (it stays
// in BF16 under mixed-precision quantisation: "SANA-Streaming：基于混合扩散
// Transformer的实时流式视频编辑系统", 实验结果) without writing its activations;
// the maps taken are the plainest ones onto the scan's ranges g <= 0 and
// beta in (0, 1):  g = -softplus(x) = -log(1 + e^x),  beta = sigmoid(y).
#pragma once

namespace gdn {

// -softplus(x), formed without overflow: -(max(x, 0) + log1p(e^{-|x|})).
__device__ __forceinline__ float gate_g_from_logit(float x) {
  return -(fmaxf(x, 0.f) + log1pf(expf(-fabsf(x))));
}

// sigmoid(y) = 1 / (1 + e^{-y}); e^{-y} overflowing to inf gives 0.
__device__ __forceinline__ float gate_beta_from_logit(float y) { return 1.f / (1.f + expf(-y)); }

}  // namespace gdn

// la_state.cuh -- combining the states of consecutive chunks of a sequence.
//
// The recurrence S_t = gamma S_{t-1} + k_t^T v_t ("MiniMax-M1" model entry,
// linear/SSM layer field: per-head exponential decay, 128x128 state per head)
// is linear in its initial state, so the state after R consecutive chunks of
// n_0, ..., n_{R-1} tokens is
//     S = gamma^(n_0 + ... + n_{R-1}) S_0 + sum_j gamma^(n_{j+1} + ... + n_{R-1}) L_j
// where L_j is chunk j's state from a zero initial state (lightning_attn_state
// with no initial state).  This is the exchange step that lets one sequence be
// split across GPUs (each rank computes the L_j of its own chunk, the L_j are
// all-gathered, and each rank combines those before its chunk into its
// entering state) -- the long-context inference of the MiniMax-01 abstract (4M
// tokens).  Evaluated by Horner's rule, S <- gamma^(n_j) S + L_j, one float4
// of one head per thread: a read of R + 1 states and a write of one, HBM-bound.
#pragma once

#include <stdint.h>

namespace la {

constexpr int COMBINE_MAX_CHUNKS = 256;

struct CombineArgs {
  const float* states;  // [R][nseq][D*E]
  const float* init;    // nullable [nseq][D*E]
  const float* slopes;  // [H]
  float* out;           // [nseq][D*E]
  int64_t per_seq4;     // D*E / 4
  int64_t total4;       // nseq * D*E / 4
  int H, R;
  int n[COMBINE_MAX_CHUNKS];  // chunk token counts
};

__global__ void __launch_bounds__(256) state_combine_kernel(const CombineArgs a) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < a.total4;
       i += stride) {
    const int64_t seq = i / a.per_seq4;
    const float lam = a.slopes[seq % a.H];
    float4 s = a.init ? __ldg(reinterpret_cast<const float4*>(a.init) + i)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < a.R; ++j) {
      const float g = expf(-lam * static_cast<float>(a.n[j]));
      const float4 l = __ldg(reinterpret_cast<const float4*>(a.states) + j * a.total4 + i);
      s.x = fmaf(g, s.x, l.x);
      s.y = fmaf(g, s.y, l.y);
      s.z = fmaf(g, s.z, l.z);
      s.w = fmaf(g, s.w, l.w);
    }
    reinterpret_cast<float4*>(a.out)[i] = s;
  }
}

}  // namespace la

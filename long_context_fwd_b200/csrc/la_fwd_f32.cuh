// la_fwd_f32.cuh -- fp32 Lightning Attention prefill on CUDA cores.
//
// For fp32 inputs and fp32-class accuracy (bf16 tensor-core operands would
// not meet it).  One CTA per (b, h) walks the sequence in blocks of BT = 32
// tokens with the fp32 D x E state in shared memory.  For the block
// [t0, t0 + len) with local rows i, j:
//   P_ij   = (q_i . k_j) gamma^(i - j)          for j <= i   (intra scores)
//   o_i    = gamma^(i+1) q_i S + sum_j P_ij v_j (inter through the state + intra)
//   S     <- gamma^len S + sum_j gamma^(len-1-j) k_j^T v_j   (state carry)
// which is the definition o_t = sum_{s<=t} gamma^(t-s) (q_t . k_s) v_s split at
// block boundaries ("MiniMax-M1" model entry (archdb), linear/SSM layer field:
// per-head exponential decay and a fixed-size per-head state).  All decay
// factors are gamma^m with 0 <= m <= BT, so none exceeds 1.
#pragma once

#include <stdint.h>

namespace la {

constexpr int F32_BT = 32;

template <int D, int E>
__host__ __device__ constexpr size_t fwd_f32_smem_bytes() {
  return sizeof(float) * (size_t)(D * E + F32_BT * D + F32_BT * (D + 1) + F32_BT * E +
                                  F32_BT * (F32_BT + 1) + (F32_BT + 1));
}

template <int D, int E>
__global__ void __launch_bounds__(256) fwd_f32_kernel(const float* __restrict__ q,
                                                      const float* __restrict__ k,
                                                      const float* __restrict__ v,
                                                      const float* __restrict__ slopes,
                                                      float* __restrict__ out, int H, int N) {
  constexpr int BT = F32_BT, T = 256;
  extern __shared__ float smf[];
  float* KV = smf;                   // [D][E]
  float* Qs = KV + D * E;            // [BT][D]
  float* Ks = Qs + BT * D;           // [BT][D + 1] (padded: column reads conflict-free)
  float* Vs = Ks + BT * (D + 1);     // [BT][E]
  float* P = Vs + BT * E;            // [BT][BT + 1]
  float* pw = P + BT * (BT + 1);     // gamma^m, m = 0..BT

  const int tid = threadIdx.x;
  const int64_t bh = blockIdx.x;
  const float lam = slopes[bh % H];
  const float* qb = q + bh * (int64_t)N * D;
  const float* kb = k + bh * (int64_t)N * D;
  const float* vb = v + bh * (int64_t)N * E;
  float* ob = out + bh * (int64_t)N * E;

  for (int i = tid; i < D * E; i += T) KV[i] = 0.f;
  for (int i = tid; i <= BT; i += T) pw[i] = expf(-lam * static_cast<float>(i));

  for (int t0 = 0; t0 < N; t0 += BT) {
    const int len = min(BT, N - t0);
    __syncthreads();  // previous block finished reading the tiles and the state
    for (int i = tid; i < BT * D; i += T) {
      const int r = i / D, c = i % D;
      const bool in = r < len;
      Qs[i] = in ? qb[(int64_t)(t0 + r) * D + c] : 0.f;
      Ks[r * (D + 1) + c] = in ? kb[(int64_t)(t0 + r) * D + c] : 0.f;
    }
    for (int i = tid; i < BT * E; i += T) {
      const int r = i / E, c = i % E;
      Vs[i] = r < len ? vb[(int64_t)(t0 + r) * E + c] : 0.f;
    }
    __syncthreads();
    for (int i = tid; i < BT * BT; i += T) {
      const int r = i / BT, j = i % BT;
      float p = 0.f;
      if (j <= r && r < len) {
        float dot = 0.f;
#pragma unroll 8
        for (int d = 0; d < D; ++d) dot = fmaf(Qs[r * D + d], Ks[j * (D + 1) + d], dot);
        p = dot * pw[r - j];
      }
      P[r * (BT + 1) + j] = p;
    }
    __syncthreads();
    for (int i = tid; i < BT * E; i += T) {
      const int r = i / E, e = i % E;
      if (r < len) {
        float a = 0.f;
#pragma unroll 8
        for (int d = 0; d < D; ++d) a = fmaf(Qs[r * D + d], KV[d * E + e], a);
        float b = 0.f;
        for (int j = 0; j <= r; ++j) b = fmaf(P[r * (BT + 1) + j], Vs[j * E + e], b);
        ob[(int64_t)(t0 + r) * E + e] = fmaf(pw[r + 1], a, b);
      }
    }
    __syncthreads();  // the state is read above before it is updated below
    for (int i = tid; i < D * E; i += T) {
      const int d = i / E, e = i % E;
      float a = 0.f;
      for (int j = 0; j < len; ++j) a = fmaf(pw[len - 1 - j] * Ks[j * (D + 1) + d], Vs[j * E + e], a);
      KV[i] = fmaf(pw[len], KV[i], a);
    }
  }
}

}  // namespace la

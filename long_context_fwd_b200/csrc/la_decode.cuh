// la_decode.cuh -- one recurrent Lightning Attention decode step (CUDA cores).
//
// Per (b, h):  S <- gamma S + k^T v ;  o = q S      (gamma = exp(-lambda_h))
// the fixed-size recurrent state of the linear layers ("MiniMax-M1" model entry
// (archdb): layers with a fixed-size recurrent state; linear/SSM layer field:
// per-head exponential decay, 128x128 state per head).
//
// The step is a read-modify-write of the fp32 D x E state (64 KiB per head at
// D = E = 128): HBM-bound.  One CTA of 256 threads per (b, h); each warp
// streams whole 512-byte state rows with 128-bit loads/stores (evict-first),
// each thread updates 4 columns of D/8 rows and accumulates its share of q.S;
// an 8-way shared-memory reduction finishes o.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace la {

template <int D, int E>
__global__ void __launch_bounds__(256) decode_kernel(const __nv_bfloat16* __restrict__ q,
                                                     const __nv_bfloat16* __restrict__ k,
                                                     const __nv_bfloat16* __restrict__ v,
                                                     float* __restrict__ state,
                                                     const float* __restrict__ slopes,
                                                     float* __restrict__ out, int H) {
  constexpr int T = 256;
  constexpr int C4 = E / 4;      // threads per state row (one float4 each)
  constexpr int RPI = T / C4;    // rows covered per pass
  constexpr int R = D / RPI;     // rows per thread
  static_assert(R * RPI == D && C4 * RPI == T, "unsupported head geometry");

  __shared__ float sq[D];
  __shared__ float sk[D];
  __shared__ float red[RPI][E];

  const int tid = threadIdx.x;
  const int64_t bh = blockIdx.x;
  const int h = static_cast<int>(bh % H);
  const int c4 = tid % C4;
  const int r0 = tid / C4;

  float4* S = reinterpret_cast<float4*>(state + bh * (int64_t)(D * E));
  float4 s[R];
#pragma unroll
  for (int r = 0; r < R; ++r) s[r] = __ldcs(S + (r0 + r * RPI) * C4 + c4);

  for (int i = tid; i < D; i += T) {
    sq[i] = __bfloat162float(q[bh * D + i]);
    sk[i] = __bfloat162float(k[bh * D + i]);
  }
  const uint2 vr = *reinterpret_cast<const uint2*>(v + bh * E + 4 * c4);
  const float v0 = __uint_as_float(vr.x << 16), v1 = __uint_as_float(vr.x & 0xFFFF0000u);
  const float v2 = __uint_as_float(vr.y << 16), v3 = __uint_as_float(vr.y & 0xFFFF0000u);
  const float g = expf(-slopes[h]);
  __syncthreads();

  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int d = r0 + r * RPI;
    const float kd = sk[d], qd = sq[d];
    float4 t = s[r];
    t.x = fmaf(g, t.x, kd * v0);
    t.y = fmaf(g, t.y, kd * v1);
    t.z = fmaf(g, t.z, kd * v2);
    t.w = fmaf(g, t.w, kd * v3);
    __stcs(S + d * C4 + c4, t);
    a0 = fmaf(qd, t.x, a0);
    a1 = fmaf(qd, t.y, a1);
    a2 = fmaf(qd, t.z, a2);
    a3 = fmaf(qd, t.w, a3);
  }
  *reinterpret_cast<float4*>(&red[r0][4 * c4]) = make_float4(a0, a1, a2, a3);
  __syncthreads();
  if (tid < E) {
    float o = 0.f;
#pragma unroll
    for (int rr = 0; rr < RPI; ++rr) o += red[rr][tid];
    out[bh * E + tid] = o;
  }
}

}  // namespace la

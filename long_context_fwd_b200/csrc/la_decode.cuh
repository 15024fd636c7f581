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

namespace la {

// One decode step of the layer around the operator ("MiniMax-M1" model entry,
// linear-layer field: SiLU on Q, K, V and RMSNorm on the output; gate field: a
// sigmoid gate after the RMSNorm), per (b, h):
//   S <- gamma S + silu(k)^T silu(v) ;  o = silu(q) S ;
//   y = w_h * o / sqrt(mean_e(o_e^2) + eps) * sigmoid(gate)      (bf16 out)
// Same state traffic and thread layout as decode_kernel; the activations and
// the norm are a few hundred CUDA-core operations per head on top of the
// 64 KiB state read-modify-write, so the step stays HBM-bound.  Three CTAs per
// SM (at most 85 registers, as decode_kernel's 80 allow): with two, the
// 256 x 64 heads step took 0.363-0.374 ms instead of 0.322-0.328 ms.  q, k, v, gate
// and out are addressed through {b, h} element strides (a token's projections
// may sit in one fused buffer); the state is contiguous [B][H][D][E].
struct DecodeLayerArgs {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const __nv_bfloat16* gate;
  float* state;
  const float* slopes;
  const float* norm_w;  // [H][E]
  __nv_bfloat16* out;
  long long qs[2], ks[2], vs[2], gs[2], os[2];  // {b, h} element strides
  float eps;
  int H;
};

__device__ __forceinline__ float silu_f(float x) { return x / (1.f + expf(-x)); }

template <int D, int E>
__global__ void __launch_bounds__(256, 3) decode_layer_kernel(const DecodeLayerArgs a) {
  constexpr int T = 256;
  constexpr int C4 = E / 4;
  constexpr int RPI = T / C4;
  constexpr int R = D / RPI;
  static_assert(R * RPI == D && C4 * RPI == T, "unsupported head geometry");

  __shared__ float sq[D];
  __shared__ float sk[D];
  __shared__ float red[RPI][E];
  __shared__ float msq[E / 32];

  const int tid = threadIdx.x;
  const int64_t bh = blockIdx.x;
  const int64_t b = bh / a.H;
  const int h = static_cast<int>(bh % a.H);
  const int c4 = tid % C4;
  const int r0 = tid / C4;

  float4* S = reinterpret_cast<float4*>(a.state + bh * (int64_t)(D * E));
  float4 s[R];
#pragma unroll
  for (int r = 0; r < R; ++r) s[r] = __ldcs(S + (r0 + r * RPI) * C4 + c4);

  const __nv_bfloat16* qrow = a.q + b * a.qs[0] + h * a.qs[1];
  const __nv_bfloat16* krow = a.k + b * a.ks[0] + h * a.ks[1];
  for (int i = tid; i < D; i += T) {
    sq[i] = silu_f(__bfloat162float(qrow[i]));
    sk[i] = silu_f(__bfloat162float(krow[i]));
  }
  const uint2 vr = *reinterpret_cast<const uint2*>(a.v + b * a.vs[0] + h * a.vs[1] + 4 * c4);
  const float v0 = silu_f(__uint_as_float(vr.x << 16));
  const float v1 = silu_f(__uint_as_float(vr.x & 0xFFFF0000u));
  const float v2 = silu_f(__uint_as_float(vr.y << 16));
  const float v3 = silu_f(__uint_as_float(vr.y & 0xFFFF0000u));
  const float g = expf(-a.slopes[h]);
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
  float o = 0.f;
  if (tid < E) {
#pragma unroll
    for (int rr = 0; rr < RPI; ++rr) o += red[rr][tid];
    float ss = o * o;
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
    if ((tid & 31) == 0) msq[tid >> 5] = ss;
  }
  __syncthreads();
  if (tid < E) {
    float ms = 0.f;
#pragma unroll
    for (int i = 0; i < E / 32; ++i) ms += msq[i];
    const float rinv = rsqrtf(ms / static_cast<float>(E) + a.eps);
    const float gt = __bfloat162float(a.gate[b * a.gs[0] + h * a.gs[1] + tid]);
    const float y = a.norm_w[static_cast<int64_t>(h) * E + tid] * o * rinv / (1.f + expf(-gt));
    a.out[b * a.os[0] + h * a.os[1] + tid] = __float2bfloat16_rn(y);
  }
}

}  // namespace la

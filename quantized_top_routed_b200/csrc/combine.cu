// Stage 5: gate-weighted unpermute and combine (and, for stage 3, the
// permutation of the activation rows into schedule order).
//   out[t] = sum_{j<k} g[t,j] * Y[inv_pos[t,j]] + sum_{s<S} Y[T*k + s*T + t]
// fp32 accumulation in slot order, then the shared experts (weight 1), one
// round to bf16 (nearest even) at the end.  ("OmniMoE: An Efficient MoE by
// Orchestrating Atomic Experts at Scale", section 2.1: the shared dense MLP is
// active for every input; "FineRMoE", Sparse Sum Layer: outputs weighted by
// the router's probabilities.)
//
// Each thread moves one 16-byte vector (8 bf16) of one token, so every Y row
// and the output row are read and written with coalesced 16-byte accesses.
#include <cuda_fp16.h>

#include "qmoe_internal.cuh"

namespace qmoe {
namespace {

__device__ __forceinline__ void acc8(float (&a)[8], const uint4 v, float g) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    a[2 * i] = fmaf(g, __uint_as_float(w[i] << 16), a[2 * i]);
    a[2 * i + 1] = fmaf(g, __uint_as_float(w[i] & 0xFFFF0000u), a[2 * i + 1]);
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&p);
}

// One thread per 16-byte output vector: all k + S row loads are issued
// before any accumulation, so a token costs one memory round trip.
__global__ void __launch_bounds__(256) combine_kernel(const uint16_t* __restrict__ Y, const float* __restrict__ gate,
                                                      const int32_t* __restrict__ inv_pos, int T, int k, int S,
                                                      int d, uint16_t* __restrict__ out, int* __restrict__ err) {
  pdl_wait();                                   // Y is complete past this point
  const int nvec = d >> 3;
  const long long gv = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (gv >= (long long)T * nvec) return;
  const int t = (int)(gv / nvec), v = (int)(gv - (long long)t * nvec);
  uint4 y[kMaxK + kMaxShared];
  float g[kMaxK];
#pragma unroll
  for (int j = 0; j < kMaxK; ++j) {
    if (j < k) {
      const int pos = __ldg(inv_pos + (size_t)t * k + j);
      g[j] = __ldg(gate + (size_t)t * k + j);
      if (dbg_in_bounds(pos >= 0 && pos < T * k, err)) {
        y[j] = __ldg(reinterpret_cast<const uint4*>(Y + (size_t)pos * d) + v);
      } else {
        y[j] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
  }
#pragma unroll
  for (int s = 0; s < kMaxShared; ++s)
    if (s < S) y[kMaxK + s] = __ldg(reinterpret_cast<const uint4*>(Y + ((size_t)T * k + (size_t)s * T + t) * d) + v);
  float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int j = 0; j < kMaxK; ++j)
    if (j < k) acc8(a, y[j], g[j]);
#pragma unroll
  for (int s = 0; s < kMaxShared; ++s)
    if (s < S) acc8(a, y[kMaxK + s], 1.0f);
  uint4 o;
  o.x = pack_bf16x2(a[0], a[1]);
  o.y = pack_bf16x2(a[2], a[3]);
  o.z = pack_bf16x2(a[4], a[5]);
  o.w = pack_bf16x2(a[6], a[7]);
  reinterpret_cast<uint4*>(out + (size_t)t * d)[v] = o;
}

// Activation rows in schedule order for the gate/up GEMM: one thread per
// 16-byte vector, so each row is read and written with coalesced accesses.
__global__ void __launch_bounds__(256) permute_rows_kernel(const uint16_t* __restrict__ x,
                                                           const int32_t* __restrict__ sorted_token, int P, int d,
                                                           uint16_t* __restrict__ xp, int to_f16, int T,
                                                           int* __restrict__ err) {
  pdl_wait();                                   // the schedule's permutation is complete past this point
  const int nvec = d >> 3;
  const long long gv = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (gv >= (long long)P * nvec) return;
  const int p = (int)(gv / nvec), v = (int)(gv - (long long)p * nvec);
  const int t = __ldg(sorted_token + p);
  if (!dbg_in_bounds(t >= 0 && t < T, err)) return;
  uint4 q = __ldg(reinterpret_cast<const uint4*>(x + (size_t)t * d) + v);
  if (to_f16) {                                 // bf16 -> fp16 (exact inside the fp16 range)
    uint32_t* w = reinterpret_cast<uint32_t*>(&q);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __half2 h = __floats2half2_rn(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
      w[i] = *reinterpret_cast<const uint32_t*>(&h);
    }
  }
  reinterpret_cast<uint4*>(xp + (size_t)p * d)[v] = q;
}

}  // namespace

cudaError_t launch_permute_rows(bool pdl, const uint16_t* x, const int32_t* sorted_token, int P, int d, uint16_t* xp,
                                bool to_f16, int T, int* err, cudaStream_t s) {
  const long long n = (long long)P * (d >> 3);
  return launch_ex(permute_rows_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, s, pdl, x, sorted_token, P,
                   d, xp, to_f16 ? 1 : 0, T, err);
}

cudaError_t launch_combine(bool pdl, const uint16_t* Y, const float* gate, const int32_t* inv_pos, int T, int k, int S, int d,
                           uint16_t* out, int* err, cudaStream_t s) {
  const long long n = (long long)T * (d >> 3);
  return launch_ex(combine_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, s, pdl, Y, gate, inv_pos, T, k, S,
                   d, out, err);
}

}  // namespace qmoe

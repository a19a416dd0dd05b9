// Stage 5: gate-weighted unpermute and combine.
//   out[t] = sum_{j<k} g[t,j] * Y[inv_pos[t,j]] + sum_{s<S} Y[T*k + s*T + t]
// fp32 accumulation in slot order, then the shared experts (weight 1), one
// round to bf16 (nearest even) at the end.  ("OmniMoE: An Efficient MoE by
// Orchestrating Atomic Experts at Scale", section 2.1: the shared dense MLP is
// active for every input; "FineRMoE", Sparse Sum Layer: outputs weighted by
// the router's probabilities.)
//
// One CTA per token; each thread moves 16-byte vectors (8 bf16), so every Y
// row and the output row are read/written with coalesced 16-byte accesses.
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

__global__ void __launch_bounds__(128) combine_kernel(const uint16_t* __restrict__ Y, const float* __restrict__ gate,
                                                      const int32_t* __restrict__ inv_pos, int T, int k, int S,
                                                      int d, uint16_t* __restrict__ out) {
  __shared__ float g[kMaxK];
  __shared__ int32_t pos[kMaxK];
  const int t = blockIdx.x;
  if (threadIdx.x < k) {
    g[threadIdx.x] = gate[(size_t)t * k + threadIdx.x];
    pos[threadIdx.x] = inv_pos[(size_t)t * k + threadIdx.x];
  }
  __syncthreads();
  const int nvec = d >> 3;
  for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
    float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < k; ++j) {
      const uint4 y = __ldg(reinterpret_cast<const uint4*>(Y + (size_t)pos[j] * d) + v);
      acc8(a, y, g[j]);
    }
    for (int s = 0; s < S; ++s) {
      const uint4 y = __ldg(reinterpret_cast<const uint4*>(Y + ((size_t)T * k + (size_t)s * T + t) * d) + v);
      acc8(a, y, 1.0f);
    }
    uint4 o;
    o.x = pack_bf16x2(a[0], a[1]);
    o.y = pack_bf16x2(a[2], a[3]);
    o.z = pack_bf16x2(a[4], a[5]);
    o.w = pack_bf16x2(a[6], a[7]);
    reinterpret_cast<uint4*>(out + (size_t)t * d)[v] = o;
  }
}

}  // namespace

cudaError_t launch_combine(const uint16_t* Y, const float* gate, const int32_t* inv_pos, int T, int k, int S, int d,
                           uint16_t* out, cudaStream_t s) {
  combine_kernel<<<T, 128, 0, s>>>(Y, gate, inv_pos, T, k, S, d, out);
  return cudaGetLastError();
}

}  // namespace qmoe

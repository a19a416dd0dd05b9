// Stage 1: router.  z[t,e] = sum_i x[t,i] * Wr[e,i] (+ b[e]) in fp32, then per
// token a softmax over all E logits, top-k by logit (lower expert index
// first on ties) and the selected probabilities renormalised to sum to 1.
// ("Quantized Mixture of Experts (Q-MoE)", section 3, gating network with
// top-k routing; "FineRMoE", Sparse Sum Layer: softmax probabilities as
// mixing weights.)
//
// Two kernels:
//  * router_logits_kernel: a 32-token x 32-expert fp32 tile per CTA over one
//    slice of d (d is split so the grid covers the SMs when T is small).
//    Each slice's partial sums go to zpart[slice][T][E]; the summation order
//    is fixed, so the logits are deterministic.
//  * router_topk_kernel: one warp per token; the E logits live in registers
//    (ceil(E/32) per lane), top-k is k rounds of a warp arg-max.
#include "qmoe_internal.cuh"

#include <math.h>

namespace qmoe {
namespace {

constexpr int RT = 32;   // tokens per CTA
constexpr int RE = 32;   // experts per CTA
constexpr int RC = 32;   // d elements per smem chunk
constexpr int RS = RC + 4;

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__global__ void __launch_bounds__(256) router_logits_kernel(const uint16_t* __restrict__ x,
                                                            const float* __restrict__ Wr, int T, int d,
                                                            int E, int slice, float* __restrict__ zpart) {
  __shared__ __align__(16) float xs[RT][RS];
  __shared__ __align__(16) float ws[RE][RS];
  const int t0 = blockIdx.x * RT, e0 = blockIdx.y * RE, c_begin = blockIdx.z * slice;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const int lr = tid >> 3, lc = (tid & 7) * 4;   // loader: row, column
  float acc00 = 0.f, acc01 = 0.f, acc10 = 0.f, acc11 = 0.f;  // [token ty|ty+16][expert tx|tx+16]

  for (int c0 = c_begin; c0 < c_begin + slice; c0 += RC) {
    {
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      const int t = t0 + lr;
      if (t < T) {
        const uint2 raw = *reinterpret_cast<const uint2*>(x + (size_t)t * d + c0 + lc);
        v = make_float4(bf16_lo(raw.x), bf16_hi(raw.x), bf16_lo(raw.y), bf16_hi(raw.y));
      }
      *reinterpret_cast<float4*>(&xs[lr][lc]) = v;
      float4 w = make_float4(0.f, 0.f, 0.f, 0.f);
      const int e = e0 + lr;
      if (e < E) w = *reinterpret_cast<const float4*>(Wr + (size_t)e * d + c0 + lc);
      *reinterpret_cast<float4*>(&ws[lr][lc]) = w;
    }
    __syncthreads();
#pragma unroll
    for (int c = 0; c < RC; c += 4) {
      const float4 a0 = *reinterpret_cast<const float4*>(&xs[ty][c]);
      const float4 a1 = *reinterpret_cast<const float4*>(&xs[ty + 16][c]);
      const float4 b0 = *reinterpret_cast<const float4*>(&ws[tx][c]);
      const float4 b1 = *reinterpret_cast<const float4*>(&ws[tx + 16][c]);
      acc00 = fmaf(a0.x, b0.x, acc00); acc00 = fmaf(a0.y, b0.y, acc00);
      acc00 = fmaf(a0.z, b0.z, acc00); acc00 = fmaf(a0.w, b0.w, acc00);
      acc01 = fmaf(a0.x, b1.x, acc01); acc01 = fmaf(a0.y, b1.y, acc01);
      acc01 = fmaf(a0.z, b1.z, acc01); acc01 = fmaf(a0.w, b1.w, acc01);
      acc10 = fmaf(a1.x, b0.x, acc10); acc10 = fmaf(a1.y, b0.y, acc10);
      acc10 = fmaf(a1.z, b0.z, acc10); acc10 = fmaf(a1.w, b0.w, acc10);
      acc11 = fmaf(a1.x, b1.x, acc11); acc11 = fmaf(a1.y, b1.y, acc11);
      acc11 = fmaf(a1.z, b1.z, acc11); acc11 = fmaf(a1.w, b1.w, acc11);
    }
    __syncthreads();
  }
  float* zp = zpart + (size_t)blockIdx.z * T * E;
  const int ta = t0 + ty, tb = t0 + ty + 16, ea = e0 + tx, eb = e0 + tx + 16;
  if (ta < T && ea < E) zp[(size_t)ta * E + ea] = acc00;
  if (ta < T && eb < E) zp[(size_t)ta * E + eb] = acc01;
  if (tb < T && ea < E) zp[(size_t)tb * E + ea] = acc10;
  if (tb < T && eb < E) zp[(size_t)tb * E + eb] = acc11;
}

// Warp arg-max over (value, index): larger value wins, lower index on ties.
__device__ __forceinline__ void warp_argmax(float& v, int& e) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, v, off);
    const int oe = __shfl_xor_sync(0xffffffffu, e, off);
    if (ov > v || (ov == v && oe < e)) {
      v = ov;
      e = oe;
    }
  }
}

template <int EPL>
__global__ void __launch_bounds__(256) router_topk_kernel(const float* __restrict__ zpart, int split,
                                                          const float* __restrict__ bias, int T, int E, int k,
                                                          int32_t* __restrict__ idx, float* __restrict__ gate) {
  const int t = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  float z[EPL];
  bool live[EPL];
  float m = -INFINITY;
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    const int e = lane + 32 * i;
    live[i] = e < E;
    float v = -INFINITY;
    if (live[i]) {
      v = 0.f;
      for (int s = 0; s < split; ++s) v += zpart[((size_t)s * T + t) * E + e];
      if (bias) v += bias[e];
    }
    z[i] = v;
    m = fmaxf(m, v);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  float den = 0.f;
#pragma unroll
  for (int i = 0; i < EPL; ++i)
    if (live[i]) den += expf(z[i] - m);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) den += __shfl_xor_sync(0xffffffffu, den, off);

  // k rounds of arg-max; lane j keeps slot j.
  float my_p = 0.f;
  int my_e = 0;
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int be = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      if (live[i] && (z[i] > bv || (z[i] == bv && e < be))) {
        bv = z[i];
        be = e;
      }
    }
    warp_argmax(bv, be);
#pragma unroll
    for (int i = 0; i < EPL; ++i)
      if (lane + 32 * i == be) live[i] = false;
    if (lane == j) {
      my_e = be;
      my_p = expf(bv - m) / den;
    }
  }
  float psum = lane < k ? my_p : 0.f;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, off);
  if (lane < k) {
    idx[(size_t)t * k + lane] = my_e;
    gate[(size_t)t * k + lane] = my_p / psum;
  }
}

}  // namespace

int router_split(int T, int d, int E, int num_sms) {
  const int tiles = ((T + RT - 1) / RT) * ((E + RE - 1) / RE);
  int split = 1;
  // split d while the grid is short of the SM count and slices stay >= 256
  while (tiles * split * 2 <= num_sms && d % (split * 2 * RC) == 0 && d / (split * 2) >= 256 && split < 16)
    split *= 2;
  return split;
}

cudaError_t launch_router_logits(const uint16_t* x, const float* Wr, int T, int d, int E, int split, float* zpart,
                                 cudaStream_t s) {
  dim3 grid((T + RT - 1) / RT, (E + RE - 1) / RE, split);
  router_logits_kernel<<<grid, 256, 0, s>>>(x, Wr, T, d, E, d / split, zpart);
  return cudaGetLastError();
}

cudaError_t launch_router_topk(const float* zpart, int split, const float* bias, int T, int E, int k, int32_t* idx,
                               float* gate, cudaStream_t s) {
  const int blocks = (T + 7) / 8;
  const int epl = (E + 31) / 32;
  switch (epl) {
    case 1: router_topk_kernel<1><<<blocks, 256, 0, s>>>(zpart, split, bias, T, E, k, idx, gate); break;
    case 2: router_topk_kernel<2><<<blocks, 256, 0, s>>>(zpart, split, bias, T, E, k, idx, gate); break;
    case 3:
    case 4: router_topk_kernel<4><<<blocks, 256, 0, s>>>(zpart, split, bias, T, E, k, idx, gate); break;
    default: router_topk_kernel<8><<<blocks, 256, 0, s>>>(zpart, split, bias, T, E, k, idx, gate); break;
  }
  return cudaGetLastError();
}

}  // namespace qmoe

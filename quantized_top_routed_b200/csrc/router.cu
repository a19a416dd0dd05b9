// Stage 1: router.  z[t,e] = sum_i x[t,i] * Wr[e,i] (+ b[e]) in fp32, then per
// token a softmax over all E logits, top-k by logit (lower expert index
// first on ties) and the selected probabilities renormalised to sum to 1.
// ("Quantized Mixture of Experts (Q-MoE)", section 3, gating network with
// top-k routing; "FineRMoE", Sparse Sum Layer: softmax probabilities as
// mixing weights.)
//
// From activations: router_logits_kernel computes a 32-token x 32-expert
// tile of fp32 logits over one slice of d (d is split so the grid covers the
// SMs when T is small), streaming x and Wr through a 3-stage cp.async ring,
// and writes its partial sums; then one warp per token sums the slices in a
// fixed order (so the logits are deterministic), adds the bias and takes the
// top-k -- in the layer's forward inside the same launch, by the last CTA to
// finish each token tile, otherwise in router_topk_kernel.  From supplied
// logits: router_topk_kernel alone, with one slice.
#include "qmoe_internal.cuh"

#include <math.h>

namespace qmoe {
namespace {

constexpr int RT = 32;          // tokens per CTA
constexpr int RE = 32;          // experts per CTA
constexpr int RC = 128;         // d elements per pipeline stage
constexpr int NST = 3;          // cp.async stages
constexpr int XS = RC + 8;      // bf16 row stride of the x stage (bank shift of 4 words per row)
constexpr int WS = RC + 4;      // fp32 row stride of the Wr stage
constexpr int kRouterThreads = 256;
constexpr int kSmemPipe = NST * (RT * XS * 2 + RE * WS * 4);
constexpr int kSmemRouter = kSmemPipe;
static_assert(kSmemPipe >= RT * kMaxE * 4, "the top-k tail keeps the tile's logits in the pipeline buffers");

// One warp: softmax + top-k + renormalisation of the E logits of NT tokens
// at once (the tokens' shuffle chains interleave; each token's arithmetic is
// the same as with NT = 1).  NaN logits are taken as -inf, so every pick is
// an expert index in [0, E) whatever the input (ties, -inf included, go to
// the lower index).  logit(u, e) gives the fp32 logit of expert e
// (bias included) for the warp's token u; token u's outputs go to
// idx0 + u * ld and gate0 + u * ld when u < nvalid.
template <int EPL, int NT, class LogitFn>
__device__ __forceinline__ void topk_tokens(LogitFn logit, int E, int k, int lane, int32_t* idx0, float* gate0,
                                            size_t ld, int nvalid) {
  static_assert(NT * EPL <= 32, "one bit per (token, expert slot)");
  float z[NT][EPL];
  uint32_t live = 0;                       // bit u * EPL + i: expert lane + 32 i of token u still unpicked
  float m[NT];
#pragma unroll
  for (int u = 0; u < NT; ++u) {
    m[u] = -INFINITY;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      const bool ok = e < E;
      if (ok) live |= 1u << (u * EPL + i);
      const float v = ok ? logit(u, e) : -INFINITY;
      z[u][i] = v == v ? v : -INFINITY;   // a NaN logit ranks below every number, so the picks stay valid experts
      m[u] = fmaxf(m[u], z[u][i]);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1)
#pragma unroll
    for (int u = 0; u < NT; ++u) m[u] = fmaxf(m[u], __shfl_xor_sync(0xffffffffu, m[u], off));
  float den[NT];
#pragma unroll
  for (int u = 0; u < NT; ++u) {
    den[u] = 0.f;
#pragma unroll
    for (int i = 0; i < EPL; ++i)
      if (live >> (u * EPL + i) & 1u) den[u] += expf(z[u][i] - m[u]);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1)
#pragma unroll
    for (int u = 0; u < NT; ++u) den[u] += __shfl_xor_sync(0xffffffffu, den[u], off);

  float my_p[NT];
  int my_e[NT];
#pragma unroll
  for (int u = 0; u < NT; ++u) {
    my_p[u] = 0.f;
    my_e[u] = 0;
  }
  for (int j = 0; j < k; ++j) {
    float bv[NT];
    int be[NT];
#pragma unroll
    for (int u = 0; u < NT; ++u) {
      bv[u] = -INFINITY;
      be[u] = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        if ((live >> (u * EPL + i) & 1u) && (z[u][i] > bv[u] || (z[u][i] == bv[u] && e < be[u]))) {
          bv[u] = z[u][i];
          be[u] = e;
        }
      }
    }
    // warp arg-max: larger value wins, lower index on ties
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
#pragma unroll
      for (int u = 0; u < NT; ++u) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv[u], off);
        const int oe = __shfl_xor_sync(0xffffffffu, be[u], off);
        if (ov > bv[u] || (ov == bv[u] && oe < be[u])) {
          bv[u] = ov;
          be[u] = oe;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < NT; ++u) {
#pragma unroll
      for (int i = 0; i < EPL; ++i)
        if (lane + 32 * i == be[u]) live &= ~(1u << (u * EPL + i));
      if (lane == j) {
        my_e[u] = be[u];
        my_p[u] = expf(bv[u] - m[u]) / den[u];
      }
    }
  }
  float psum[NT];
#pragma unroll
  for (int u = 0; u < NT; ++u) psum[u] = lane < k ? my_p[u] : 0.f;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1)
#pragma unroll
    for (int u = 0; u < NT; ++u) psum[u] += __shfl_xor_sync(0xffffffffu, psum[u], off);
#pragma unroll
  for (int u = 0; u < NT; ++u)
    if (u < nvalid && lane < k) {
      idx0[u * ld + lane] = my_e[u];
      gate0[u * ld + lane] = my_p[u] / psum[u];
    }
}

__device__ __forceinline__ void cp16(uint32_t dst, const void* src, uint32_t n) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}

// EPL = 0: partial logits only.  EPL > 0 (ceil(E / 32) rounded up to 1, 2,
// 4, 8): afterwards the last CTA to finish a 32-token tile (counted in
// tile_done[tile], which it resets to 0) takes those tokens' top-k itself,
// summing the slices in the same fixed order as router_topk_kernel, so the
// two paths give identical results and the second launch is saved.
template <int EPL>
__global__ void __launch_bounds__(kRouterThreads) router_logits_kernel(const uint16_t* __restrict__ x,
                                                                      const float* __restrict__ Wr, int T, int d,
                                                                      int E, int split, float* __restrict__ zpart,
                                                                      int* __restrict__ tile_done,
                                                                      const float* __restrict__ bias, int k,
                                                                      int32_t* __restrict__ idx,
                                                                      float* __restrict__ gate) {
  extern __shared__ __align__(16) uint8_t rsm[];
  uint16_t* xs = reinterpret_cast<uint16_t*>(rsm);                          // [NST][RT][XS]
  float* ws = reinterpret_cast<float*>(rsm + NST * RT * XS * 2);            // [NST][RE][WS]
  const int tt = blockIdx.x, et = blockIdx.y, sp = blockIdx.z;
  const int t0 = tt * RT, e0 = et * RE;
  const int slice = d / split, c_begin = sp * slice, nchunks = slice / RC;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  pdl_wait();                                   // x may come from the previous kernel on the stream

  auto issue = [&](int chunk, int stage) {
    const int c0 = c_begin + chunk * RC;
    const uint32_t xb = smem_u32(xs + stage * RT * XS);
    const uint32_t wb = smem_u32(ws + stage * RE * WS);
#pragma unroll
    for (int i = 0; i < (RT * RC * 2 / 16) / kRouterThreads; ++i) {  // x: 16 chunks of 16 B per row
      const int v = tid + i * kRouterThreads, row = v >> 4, c = v & 15;
      const int t = t0 + row;
      cp16(xb + (row * XS + c * 8) * 2, x + (size_t)min(t, T - 1) * d + c0 + c * 8, t < T ? 16 : 0);
    }
#pragma unroll
    for (int i = 0; i < (RE * RC * 4 / 16) / kRouterThreads; ++i) {  // Wr: 32 chunks of 16 B per row
      const int v = tid + i * kRouterThreads, row = v >> 5, c = v & 31;
      const int e = e0 + row;
      cp16(wb + (row * WS + c * 4) * 4, Wr + (size_t)min(e, E - 1) * d + c0 + c * 4, e < E ? 16 : 0);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };

  float acc00 = 0.f, acc01 = 0.f, acc10 = 0.f, acc11 = 0.f;  // [token ty|ty+16][expert tx|tx+16]
#pragma unroll
  for (int p = 0; p < NST - 1; ++p)
    if (p < nchunks) issue(p, p);
    else asm volatile("cp.async.commit_group;" ::: "memory");
  for (int c = 0; c < nchunks; ++c) {
    asm volatile("cp.async.wait_group %0;" ::"n"(NST - 2) : "memory");
    __syncthreads();
    if (c + NST - 1 < nchunks) issue(c + NST - 1, (c + NST - 1) % NST);
    else asm volatile("cp.async.commit_group;" ::: "memory");
    const uint16_t* xa = xs + (c % NST) * RT * XS + ty * XS;
    const uint16_t* xb = xa + 16 * XS;
    const float* wa = ws + (c % NST) * RE * WS + tx * WS;
    const float* wb = wa + 16 * WS;
#pragma unroll 8
    for (int i = 0; i < RC; i += 4) {
      const uint2 ua = *reinterpret_cast<const uint2*>(xa + i);
      const uint2 ub = *reinterpret_cast<const uint2*>(xb + i);
      const float4 va = *reinterpret_cast<const float4*>(wa + i);
      const float4 vb = *reinterpret_cast<const float4*>(wb + i);
      const float a0 = __uint_as_float(ua.x << 16), a1 = __uint_as_float(ua.x & 0xFFFF0000u);
      const float a2 = __uint_as_float(ua.y << 16), a3 = __uint_as_float(ua.y & 0xFFFF0000u);
      const float b0 = __uint_as_float(ub.x << 16), b1 = __uint_as_float(ub.x & 0xFFFF0000u);
      const float b2 = __uint_as_float(ub.y << 16), b3 = __uint_as_float(ub.y & 0xFFFF0000u);
      acc00 = fmaf(a0, va.x, acc00); acc00 = fmaf(a1, va.y, acc00);
      acc00 = fmaf(a2, va.z, acc00); acc00 = fmaf(a3, va.w, acc00);
      acc01 = fmaf(a0, vb.x, acc01); acc01 = fmaf(a1, vb.y, acc01);
      acc01 = fmaf(a2, vb.z, acc01); acc01 = fmaf(a3, vb.w, acc01);
      acc10 = fmaf(b0, va.x, acc10); acc10 = fmaf(b1, va.y, acc10);
      acc10 = fmaf(b2, va.z, acc10); acc10 = fmaf(b3, va.w, acc10);
      acc11 = fmaf(b0, vb.x, acc11); acc11 = fmaf(b1, vb.y, acc11);
      acc11 = fmaf(b2, vb.z, acc11); acc11 = fmaf(b3, vb.w, acc11);
    }
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");

  float* zp = zpart + (size_t)sp * T * E;
  const int ta = t0 + ty, tb = t0 + ty + 16, ea = e0 + tx, eb = e0 + tx + 16;
  if (ta < T && ea < E) zp[(size_t)ta * E + ea] = acc00;
  if (ta < T && eb < E) zp[(size_t)ta * E + eb] = acc01;
  if (tb < T && ea < E) zp[(size_t)tb * E + ea] = acc10;
  if (tb < T && eb < E) zp[(size_t)tb * E + eb] = acc11;
  if constexpr (EPL > 0) {
    __shared__ int s_last;
    __threadfence();                            // this CTA's partials are visible device-wide
    __syncthreads();
    if (tid == 0) {
      const int contributors = (int)(gridDim.y * gridDim.z);
      const int before = atomicAdd(&tile_done[tt], 1);
      s_last = before == contributors - 1;
      if (s_last) tile_done[tt] = 0;            // every contributor has arrived: ready for the next call
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    // The tile's logits into shared memory (the pipeline buffers are free):
    // every (token, expert) pair adds its slices in ascending order, with the
    // loads of four slices of eight pairs in flight together.
    float* zs = reinterpret_cast<float*>(rsm);   // [nt][E]
    const int nt = min(RT, T - t0), np = nt * E;
    const float* zt = zpart + (size_t)t0 * E;
    const size_t sstride = (size_t)T * E;
    for (int p0 = 0; p0 < np; p0 += 8 * kRouterThreads) {
      float acc[8];
#pragma unroll
      for (int m = 0; m < 8; ++m) acc[m] = 0.f;
      int s2 = 0;
      for (; s2 + 4 <= split; s2 += 4) {
        float v[4][8];
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int m = 0; m < 8; ++m) {
            const int p = p0 + m * kRouterThreads + tid;
            v[u][m] = p < np ? __ldcg(zt + (size_t)(s2 + u) * sstride + p) : 0.f;
          }
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int m = 0; m < 8; ++m) acc[m] += v[u][m];
      }
      for (; s2 < split; ++s2)
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          const int p = p0 + m * kRouterThreads + tid;
          if (p < np) acc[m] += __ldcg(zt + (size_t)s2 * sstride + p);
        }
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const int p = p0 + m * kRouterThreads + tid;
        if (p < np) zs[p] = bias ? acc[m] + bias[p % E] : acc[m];
      }
    }
    __syncthreads();
    // warp w takes tokens w + 8u (u < 4) of the tile, all four at once
    constexpr int kWarps = kRouterThreads / 32, NT = RT / kWarps;
    const int warp = tid >> 5, lane = tid & 31;
    if (warp >= nt) return;
    const int nvalid = min(NT, (nt - warp + kWarps - 1) / kWarps);
    auto logit = [&](int u, int e) { return zs[min(warp + kWarps * u, nt - 1) * E + e]; };
    topk_tokens<EPL, NT>(logit, E, k, lane, idx + (size_t)(t0 + warp) * k, gate + (size_t)(t0 + warp) * k,
                         (size_t)kWarps * k, nvalid);
  }
}

// One warp per token: logit(e) = sum over slices s (in order) of zpart[s][t][e],
// plus the bias, then softmax, top-k and renormalisation.
template <int EPL>
__global__ void __launch_bounds__(256) router_topk_kernel(const float* __restrict__ zpart, int split,
                                                          const float* __restrict__ bias, int T, int E, int k,
                                                          int32_t* __restrict__ idx, float* __restrict__ gate) {
  pdl_wait();
  const int t = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  auto logit = [&](int, int e) {
    float acc = 0.f;
    for (int s2 = 0; s2 < split; ++s2) acc += __ldcg(zpart + ((size_t)s2 * T + t) * E + e);
    return bias ? acc + bias[e] : acc;
  };
  topk_tokens<EPL, 1>(logit, E, k, lane, idx + (size_t)t * k, gate + (size_t)t * k, (size_t)k, 1);
}

cudaError_t launch_topk(const float* zpart, int split, const float* bias, int T, int E, int k, int32_t* idx,
                        float* gate, cudaStream_t s) {
  const dim3 blocks((T + 7) / 8), threads(256);
  switch ((E + 31) / 32) {
    case 1: return launch_ex(router_topk_kernel<1>, blocks, threads, 0, s, false, zpart, split, bias, T, E, k, idx, gate);
    case 2: return launch_ex(router_topk_kernel<2>, blocks, threads, 0, s, false, zpart, split, bias, T, E, k, idx, gate);
    case 3:
    case 4: return launch_ex(router_topk_kernel<4>, blocks, threads, 0, s, false, zpart, split, bias, T, E, k, idx, gate);
    default: return launch_ex(router_topk_kernel<8>, blocks, threads, 0, s, false, zpart, split, bias, T, E, k, idx, gate);
  }
}

}  // namespace

int router_split(int T, int d, int E, int num_sms) {
  const int tiles = ((T + RT - 1) / RT) * ((E + RE - 1) / RE);
  int split = 1;
  // split d while the grid is short of the SM count and every slice keeps >= 2 stages
  while (tiles * split * 2 <= num_sms && d % (split * 2 * RC) == 0 && d / (split * 2) >= 2 * RC && split < 16)
    split *= 2;
  return split;
}

cudaError_t launch_router(const uint16_t* x, const float* Wr, const float* bias, int T, int d, int E, int k, int split,
                          float* zpart, int32_t* idx, float* gate, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(router_logits_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kSmemRouter);
  if (e != cudaSuccess) return e;
  const dim3 grid((T + RT - 1) / RT, (E + RE - 1) / RE, split);
  e = launch_ex(router_logits_kernel<0>, grid, dim3(kRouterThreads), kSmemRouter, s, false, x, Wr, T, d, E, split,
                zpart, (int*)nullptr, (const float*)nullptr, k, (int32_t*)nullptr, (float*)nullptr);
  if (e != cudaSuccess) return e;
  return launch_topk(zpart, split, bias, T, E, k, idx, gate, s);
}

namespace {
template <int EPL>
cudaError_t launch_fused(const uint16_t* x, const float* Wr, const float* bias, int T, int d, int E, int k, int split,
                         float* zpart, int* tile_done, int32_t* idx, float* gate, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(router_logits_kernel<EPL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kSmemRouter);
  if (e != cudaSuccess) return e;
  const dim3 grid((T + RT - 1) / RT, (E + RE - 1) / RE, split);
  return launch_ex(router_logits_kernel<EPL>, grid, dim3(kRouterThreads), kSmemRouter, s, false, x, Wr, T, d, E,
                   split, zpart, tile_done, bias, k, idx, gate);
}
}  // namespace

cudaError_t launch_router_fused(const uint16_t* x, const float* Wr, const float* bias, int T, int d, int E, int k,
                                int split, float* zpart, int* tile_done, int32_t* idx, float* gate, cudaStream_t s) {
  switch ((E + 31) / 32) {
    case 1: return launch_fused<1>(x, Wr, bias, T, d, E, k, split, zpart, tile_done, idx, gate, s);
    case 2: return launch_fused<2>(x, Wr, bias, T, d, E, k, split, zpart, tile_done, idx, gate, s);
    case 3:
    case 4: return launch_fused<4>(x, Wr, bias, T, d, E, k, split, zpart, tile_done, idx, gate, s);
    default: return launch_fused<8>(x, Wr, bias, T, d, E, k, split, zpart, tile_done, idx, gate, s);
  }
}

cudaError_t launch_router_topk(const float* logits, int T, int E, int k, int32_t* idx, float* gate, cudaStream_t s) {
  return launch_topk(logits, 1, nullptr, T, E, k, idx, gate, s);
}

}  // namespace qmoe

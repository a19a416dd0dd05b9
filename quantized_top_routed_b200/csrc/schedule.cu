// Stage 2: expert-centric schedule.  Every (token, slot) decision is a task;
// tasks are grouped by expert id and sorted by token id inside each group,
// so each expert's rows are contiguous for the grouped GEMMs.  ("OmniMoE: An
// Efficient MoE by Orchestrating Atomic Experts at Scale", section 2.2,
// Expert-Centric Scheduling: task collection, grouping and sorting.)
//
// One CTA of 1024 threads, deterministic (no atomics decide any position):
//   phase 1: each warp takes chunks of 32 tokens; for every expert a warp
//            ballot gives the chunk's count and each task's rank among the
//            chunk's earlier tokens;
//   phase 2: per expert, an exclusive scan of the chunk counts (the chunk's
//            base inside the expert's segment), the expert totals and the
//            exclusive scan over experts (offsets);
//   phase 3: pos(t, j) = offsets[e] + base[chunk][e] + rank; scatter.
// It also writes the segment table (routed experts, then one identity
// segment of T rows per shared expert) and, per grouped GEMM, the prefix sum
// of its tiles per segment, so the GEMMs never need the counts on the host.
#include "qmoe_internal.cuh"

namespace qmoe {
namespace {

constexpr int kThreads = 1024;
constexpr size_t kHistSmemMax = 160 * 1024;   // dynamic shared memory for chunk histograms

__device__ __forceinline__ int warp_incl_scan(int v, int lane) {
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, v, off);
    if (lane >= off) v += o;
  }
  return v;
}

__global__ void __launch_bounds__(kThreads, 1)
    schedule_kernel(const int32_t* __restrict__ idx, int T, int k, int E, int S, int bn, int mb3, int mb4,
                    const int32_t* __restrict__ seg_fmt, int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                    int32_t* __restrict__ sorted_token, int32_t* __restrict__ inv_pos,
                    int32_t* __restrict__ seg_off, int32_t* __restrict__ seg_cnt, int32_t* __restrict__ tiles,
                    int32_t* __restrict__ hist_global, int hist_in_smem, int* __restrict__ err) {
  extern __shared__ int32_t hist_smem[];
  __shared__ uint32_t bal[32][kMaxE];
  __shared__ int32_t s_cnt[kMaxE + kMaxShared];
  __shared__ int32_t s_off[kMaxE + 1];
  __shared__ int32_t s_fmt[kMaxE + kMaxShared];
  int32_t* hist = hist_in_smem ? hist_smem : hist_global;   // [C][E]: chunk counts, then chunk bases
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_wait();                                   // the router's indices are complete past this point
  const int C = (T + 31) / 32;
  const uint32_t lt_mask = (1u << lane) - 1u;

  // ---- phase 1: per-chunk counts and in-chunk ranks ------------------------
  for (int c = warp; c < C; c += 32) {
    const int t = c * 32 + lane;
    const bool valid = t < T;
    int my[kMaxK];
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      my[j] = (valid && j < k) ? idx[(size_t)t * k + j] : -1;
      if (valid && j < k && !dbg_in_bounds(my[j] >= 0 && my[j] < E, err)) my[j] = -1;
    }
    for (int w0 = 0; w0 < E; w0 += 32) {
      uint32_t m = 0;
#pragma unroll
      for (int j = 0; j < kMaxK; ++j) {
        const int e = my[j] - w0;
        if (e >= 0 && e < 32) m |= 1u << e;
      }
      uint32_t mine = 0;
#pragma unroll 8
      for (int b = 0; b < 32; ++b) {
        const uint32_t v = __ballot_sync(0xffffffffu, (m >> b) & 1u);
        if (lane == b) mine = v;
      }
      if (w0 + lane < E) {
        bal[warp][w0 + lane] = mine;
        hist[c * E + w0 + lane] = __popc(mine);
      }
    }
    __syncwarp();
#pragma unroll
    for (int j = 0; j < kMaxK; ++j)
      if (my[j] >= 0) inv_pos[(size_t)t * k + j] = __popc(bal[warp][my[j]] & lt_mask);  // rank for now
    __syncwarp();
  }
  __syncthreads();

  // ---- phase 2: chunk bases per expert, expert totals, offsets -------------
  for (int e = warp; e < E; e += 32) {
    const int per = (C + 31) / 32;
    const int c0 = min(C, lane * per), c1 = min(C, c0 + per);
    int sum = 0;
    for (int c = c0; c < c1; ++c) sum += hist[c * E + e];
    const int incl = warp_incl_scan(sum, lane);
    int run = incl - sum;
    for (int c = c0; c < c1; ++c) {
      const int h = hist[c * E + e];
      hist[c * E + e] = run;
      run += h;
    }
    if (lane == 31) s_cnt[e] = incl;
  }
  __syncthreads();
  if (warp == 0) {
    int running = 0;
    for (int e0 = 0; e0 < E; e0 += 32) {
      const int v = (e0 + lane < E) ? s_cnt[e0 + lane] : 0;
      const int incl = warp_incl_scan(v, lane);
      if (e0 + lane < E) s_off[e0 + lane] = running + incl - v;
      running += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) s_off[E] = running;
  }
  __syncthreads();

  // ---- phase 3: scatter -----------------------------------------------------
  const int P = T * k;
  for (int p = tid; p < P; p += kThreads) {
    const int t = p / k;
    const int e = idx[p];
    if (!dbg_in_bounds(e >= 0 && e < E, err)) continue;
    const int pos = s_off[e] + hist[(t >> 5) * E + e] + inv_pos[p];
    if (!dbg_in_bounds(pos >= 0 && pos < P, err)) continue;
    sorted_token[pos] = t;
    inv_pos[p] = pos;
  }
  for (int e = tid; e < E; e += kThreads) counts[e] = s_cnt[e];
  for (int e = tid; e <= E; e += kThreads) offsets[e] = s_off[e];
  for (int p = tid; p < S * T; p += kThreads) sorted_token[P + p] = p % T;

  // ---- segment and tile tables for the grouped GEMMs ------------------------
  // One prefix-sum table per (matrix, weight format): segments of another
  // format contribute no tiles, so each per-format launch walks only its own.
  if (seg_off == nullptr) return;
  const int n_seg = E + S;
  for (int e = tid; e < n_seg; e += kThreads) {
    seg_off[e] = e < E ? s_off[e] : P + (e - E) * T;
    seg_cnt[e] = e < E ? s_cnt[e] : T;
  }
  for (int e = tid; e < n_seg; e += kThreads) s_fmt[e] = seg_fmt[e];
  __syncthreads();
  if (warp < 6) {                       // warp w: matrix w / 3, format w % 3 + 1
    const int mat = warp / 3, fmt = warp % 3 + 1;
    const int mb = mat == 0 ? mb3 : mb4;
    int32_t* tab = tiles + tile_table_offset(mat, fmt, n_seg);
    int run = 0;
    for (int e0 = 0; e0 < n_seg; e0 += 32) {
      const int e = e0 + lane;
      int t = 0;
      if (e < n_seg && s_fmt[e] == fmt) {
        const int cnt = e < E ? s_cnt[e] : T;
        t = ((cnt + bn - 1) / bn) * mb;
      }
      const int incl = warp_incl_scan(t, lane);
      if (e < n_seg) tab[e] = run + incl - t;
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) tab[n_seg] = run;
  }
}

}  // namespace

size_t schedule_scratch_ints(int max_tokens, int E) { return (size_t)((max_tokens + 31) / 32) * E; }

cudaError_t launch_schedule(bool pdl, const int32_t* idx, int T, int k, int E, int S, int bn, int mb3, int mb4,
                            const int32_t* seg_fmt, int32_t* counts, int32_t* offsets, int32_t* sorted_token,
                            int32_t* inv_pos, int32_t* seg_off, int32_t* seg_cnt, int32_t* tiles, int32_t* scratch,
                            int* err, cudaStream_t s) {
  // chunk histograms live in shared memory when they fit next to the static arrays
  const size_t hist_bytes = (size_t)((T + 31) / 32) * E * sizeof(int32_t);
  const int in_smem = hist_bytes <= kHistSmemMax;
  const size_t dyn = in_smem ? hist_bytes : 0;
  if (in_smem) {
    cudaError_t e = cudaFuncSetAttribute(schedule_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kHistSmemMax);
    if (e != cudaSuccess) return e;
  }
  return launch_ex(schedule_kernel, dim3(1), dim3(kThreads), dyn, s, pdl, idx, T, k, E, S, bn, mb3, mb4, seg_fmt,
                   counts, offsets, sorted_token, inv_pos, seg_off, seg_cnt, tiles, scratch, in_smem, err);
}

}  // namespace qmoe

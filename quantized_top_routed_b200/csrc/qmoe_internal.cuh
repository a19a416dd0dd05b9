// Internal declarations and sm_100a PTX wrappers for libqmoe.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <cuda.h>

#include "../../include/qmoe.h"

namespace qmoe {

constexpr int kMaxE = 256;        // routed experts
constexpr int kMaxK = 16;         // experts per token
constexpr int kMaxShared = 8;     // shared experts
constexpr int kBK = 128;          // K elements per pipeline stage of the grouped GEMMs
constexpr int kTileM = 128;       // weight rows per GEMM tile (MMA M)

// Error bits written to the handle's device error word.
constexpr int kErrTimeout = 1;
constexpr int kErrBounds = 2;

// Bounds check of the QMOE_DEBUG build: when `ok` is false the handle's
// error word gets kErrBounds and the caller skips the access.  In the normal
// build the check is the constant true and costs nothing.
#ifdef QMOE_DEBUG
__device__ __forceinline__ bool dbg_in_bounds(bool ok, int* err) {
  if (!ok && err) atomicOr(err, kErrBounds);
  return ok;
}
#else
__device__ __forceinline__ bool dbg_in_bounds(bool, int*) { return true; }
#endif

// One expert's weights after repacking (device pointers, owned by the handle).
// mat 0 = gate/up (W13, K = d), mat 1 = down (W2, K = I).
struct ExpertDev {
  const uint8_t* w[2];     // tile blobs: [m_block][k_stage] of stage_bytes(fmt)
  const float* spc[2];     // per-channel scales in tile-row order (INT8 / FP8), else nullptr
  int32_t fmt;
  int32_t pad;
};

// Internal code of FP8 e4m3 weights when the whole layer computes in fp16:
// the codes convert to fp16 with one hardware instruction per pair, and the
// activations and H are then fp16 too (an MMA takes one input type).  Same
// tile layout as QMOE_W_FP8_E4M3_PC except the byte order inside a word.
constexpr int kFmtFp8F16 = 4;

// Bytes of one repacked (128 rows x 128 K) tile.  INT4 tiles carry their
// 128 bf16 group scales after the codes.
__host__ __device__ inline int stage_bytes(int fmt) {
  return fmt == QMOE_W_INT4_G128 ? (128 * 64 + 256) : (128 * 128);
}

// Position of K stage ks among the KS stages of a repacked 128-row block:
// the even stages first (in order), then the odd ones.
__host__ __device__ inline int stage_position(int ks, int KS) {
  return (ks & 1) ? ((KS + 1) >> 1) + (ks >> 1) : (ks >> 1);
}

// Arguments of the grouped GEMM kernels.
struct GemmArgs {
  const ExpertDev* experts;   // [n_seg]
  int mat;                    // 0: gate/up (gated SwiGLU epilogue), 1: down
  const uint16_t* act;        // B operand rows (bf16) in schedule order: permuted x [P][d] or H [P][I]
  int act_ld;                 // elements per act row
  const int32_t* seg_off;     // [n_seg] first permuted row of each segment
  const int32_t* seg_cnt;     // [n_seg] rows in each segment
  const int32_t* tile_off;    // [n_seg + 1] prefix sum of tiles per segment
  int n_seg;
  int K;                      // reduction length (d or I)
  int MB;                     // 128-row weight blocks per expert matrix
  uint16_t* out;              // H [P][I] or Y [P][d]
  int out_ld;
  int rows;                   // rows of act and out (T * (k + shared))
  int* err;                   // device error word
  long long wait_limit;       // SM cycles a bounded wait may last before the kernel aborts
};

// Default bound of every mbarrier wait in the grouped GEMMs (about a second).
constexpr long long kWaitLimit = 1ll << 31;

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar_addr, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar_addr), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking probe of the phase (test_wait never suspends the warp).
__device__ __forceinline__ bool mbar_test_wait(uint32_t bar_addr, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar_addr), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait with a suspend-time hint (ns): the warp sleeps in hardware until
// the phase completes or the hint passes, so waiting roles take no issue slots.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar_addr, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar_addr), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Slow path of mbar_wait: sleep-wait with a bound.  Gives up (returns false)
// when *abort is raised by another role or once `limit` SM cycles have
// passed, in which case it raises *abort itself.  The sleep hint is only a
// hint (the warp may sleep until the phase completes), so the time is
// checked after every return of try_wait: a wait that outlived the bound
// counts as timed out even if its phase completed meanwhile.
static __device__ __noinline__ bool mbar_wait_slow(uint32_t addr, uint32_t parity, volatile int* abort,
                                                   long long limit) {
  const long long t0 = clock64();
  const long long h = limit / 4;
  const uint32_t hint = h > 10000000ll ? 10000000u : (h < 64 ? 64u : (uint32_t)h);
  for (;;) {
    const bool done = mbar_try_wait_sleep(addr, parity, hint);
    if (clock64() - t0 > limit) {
      *abort = 1;
      return false;
    }
    if (done) return true;
    if (*abort) return false;
  }
}

// Bounded wait for the phase with the given parity.  The inline first probe
// is test_wait, which never suspends: a blocking try_wait may sleep until the
// phase completes, past any bound, so an incomplete phase always goes to the
// bounded slow path.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort, long long limit) {
  const uint32_t addr = smem_u32(bar);
  if (mbar_test_wait(addr, parity)) return true;
  return mbar_wait_slow(addr, parity, abort, limit);
}

// Bounded wait that sleeps ns nanoseconds between polls: for roles whose
// waits are long and off the critical path, so that their polling leaves the
// issue slots to the warps doing the work.
static __device__ __noinline__ bool mbar_wait_backoff_slow(uint32_t addr, uint32_t parity, volatile int* abort,
                                                           uint32_t ns, long long limit) {
  const long long t0 = clock64();
  for (;;) {
    if (mbar_test_wait(addr, parity)) return true;
    if (*abort) return false;
    if (clock64() - t0 > limit) {
      *abort = 1;
      return false;
    }
    __nanosleep(ns);
  }
}
__device__ __forceinline__ bool mbar_wait_backoff(uint64_t* bar, uint32_t parity, volatile int* abort, uint32_t ns,
                                                  long long limit) {
  const uint32_t addr = smem_u32(bar);
  if (mbar_test_wait(addr, parity)) return true;
  return mbar_wait_backoff_slow(addr, parity, abort, ns, limit);
}

// Same, ignoring the abort flag (used while draining on the way out).
__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity) {
  const uint32_t addr = smem_u32(bar);
  const long long t0 = clock64();
  while (!mbar_try_wait(addr, parity)) {
    if (clock64() - t0 > (1ll << 30)) return false;
  }
  return true;
}

// 1-D bulk copy global -> shared, completion counted on an mbarrier (bytes).
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// 16-byte cp.async with zero fill of the bytes beyond src_bytes (0 or 16).
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}

__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// --- programmatic dependent launch ------------------------------------------
// A kernel launched with launch_ex(pdl = true) may start while its
// predecessor on the stream is finishing; pdl_wait() blocks until that
// predecessor has completed and its memory is visible, so every kernel calls
// it before reading what the previous kernel wrote.  (A no-op without PDL.)
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// --- tcgen05 ---------------------------------------------------------------
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Whole warp: allocate ncols TMEM columns, address written to *slot.
__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T, kind::f16 (bf16 inputs, fp32 accumulate).
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// The same MMA and commit for a warp that executes the call together
// (warp-uniform control flow): elect.sync picks the issuing lane.  With all 32
// lanes active it elects the same lane every time, so a commit tracks the
// MMAs issued before it by this warp.
__device__ __forceinline__ void mma_bf16_ts_elect(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                                  uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t.reg .b32 r;\n\t"
      "elect.sync r|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_commit_elect(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t.reg .b32 r;\n\t"
      "elect.sync r|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(smem_u32(bar))
      : "memory");
}

// Arrive on an mbarrier once all previously issued tcgen05 ops of this thread complete.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 32 lanes x 16 consecutive 32-bit columns -> 16 registers per thread.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

// 16 registers per thread -> 32 lanes x 16 consecutive columns.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// Instruction descriptor, kind::f16: bf16 A and B (both K-major), fp32 D, M = 128.
__host__ __device__ constexpr uint32_t idesc_bf16_m128(int n, bool f16 = false) {
  return (1u << 4)                          // D format: f32
         | ((f16 ? 0u : 1u) << 7)           // A format: bf16 (1) or f16 (0)
         | ((f16 ? 0u : 1u) << 10)          // B format: the same type as A
         | ((uint32_t)(n >> 3) << 17)       // N / 8
         | ((uint32_t)(128 >> 4) << 24);    // M / 16
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (the stage buffers are 1024-byte aligned).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu)   // start address
         | ((uint64_t)1 << 16)                // leading byte offset (unused with swizzle)
         | ((uint64_t)(1024 >> 4) << 32)      // stride byte offset
         | ((uint64_t)1 << 46)                // descriptor version (sm_100)
         | ((uint64_t)2 << 61);               // SWIZZLE_128B
}

// ---------------------------------------------------------------------------
// host-side launchers (implemented in the .cu files)
// ---------------------------------------------------------------------------
// Launch kern<<<grid, block, smem, s>>>(args...), optionally as a
// programmatic dependent launch of the preceding kernel on s.
template <typename... KArgs, typename... Args>
cudaError_t launch_ex(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool pdl,
                      Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

cudaError_t launch_router(const uint16_t* x, const float* Wr, const float* bias, int T, int d, int E, int k,
                          int split, float* zpart, int32_t* idx, float* gate, cudaStream_t s);
cudaError_t launch_router_topk(const float* logits, int T, int E, int k, int32_t* idx, float* gate, cudaStream_t s);
// launch_router in one launch: tile_done holds ceil(T / 32) counters that are
// zero before the call and are zero again after it.
cudaError_t launch_router_fused(const uint16_t* x, const float* Wr, const float* bias, int T, int d, int E, int k,
                                int split, float* zpart, int* tile_done, int32_t* idx, float* gate, cudaStream_t s);
int router_split(int T, int d, int E, int num_sms);

// Tile tables written by the schedule kernel: for matrix m (0 gate/up, 1
// down) and weight format f (1..3), tiles + tile_table_offset(m, f, n_seg)
// holds the n_seg + 1 prefix sums of the tiles of the segments in format f.
__host__ __device__ inline int tile_table_offset(int mat, int fmt, int n_seg) {
  return (mat * 3 + (fmt - 1)) * (n_seg + 1);
}

cudaError_t launch_schedule(bool pdl, const int32_t* idx, int T, int k, int E, int S, int bn, int mb3, int mb4,
                            const int32_t* seg_fmt, int32_t* counts, int32_t* offsets, int32_t* sorted_token,
                            int32_t* inv_pos, int32_t* seg_off, int32_t* seg_cnt, int32_t* tiles, int32_t* scratch,
                            int* err, cudaStream_t s);
size_t schedule_scratch_ints(int max_tokens, int E);

bool gemm_bn_supported(int bn);

cudaError_t launch_grouped_gemm(bool pdl, const GemmArgs& a, const CUtensorMap& act_map, int fmt, int bn, int num_sms,
                                cudaStream_t s);

// xp[p] = x[sorted_token[p]] for p < P (activation rows in schedule order).
// to_f16: write the rows as fp16 (the fp16 MMA mode) instead of copying bf16.
cudaError_t launch_permute_rows(bool pdl, const uint16_t* x, const int32_t* sorted_token, int P, int d, uint16_t* xp,
                                bool to_f16, int T, int* err, cudaStream_t s);

cudaError_t launch_combine(bool pdl, const uint16_t* Y, const float* gate, const int32_t* inv_pos, int T, int k, int S,
                           int d, uint16_t* out, int* err, cudaStream_t s);

cudaError_t launch_repack(int fmt, int mat, const void* w, const void* scale, int rows, int K, int I,
                          uint8_t* dst, float* dst_spc, cudaStream_t s);

}  // namespace qmoe

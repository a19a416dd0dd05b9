// Stages 3-4: grouped GEMMs over the expert-centric schedule with in-kernel
// dequantisation.  ("OmniMoE: An Efficient MoE by Orchestrating Atomic
// Experts at Scale", section 2.2, Grouped GEMM: each expert's weight block is
// loaded once and reused for all of its tokens; "Quantized Mixture of
// Experts (Q-MoE)", sections 2-4: per-expert INT8 / FP8 / INT4 precision;
// "FineRMoE", architecture paragraph: gate, up and down matrices with an
// activation.)
//
//   mat 0 (gate/up): H[p, i] = silu(sum_c x[tok(p), c] W1[i, c]) * (sum_c x[tok(p), c] W3[i, c])
//   mat 1 (down):    Y[p, n] = sum_i H[p, i] W2[n, i]
//
// Layout of the contraction on the tensor cores (tcgen05, kind::f16, M=128):
//   A (M x K) = 128 weight rows, dequantised to bf16 by CUDA cores and
//               written straight into tensor memory (tcgen05.st);
//   B (N x K) = BN consecutive rows of the expert's segment in the permuted
//               activations (x rows in schedule order, or H), loaded by TMA
//               tiles (two per K stage) into 128-byte-swizzled shared memory;
//   D (M x N) = fp32 accumulators in tensor memory, double buffered.
// Weights are the M side because an expert usually has few tokens: the
// weight stream is what the kernel moves.  Raw code tiles arrive by TMA bulk
// copy into a ring sized per weight format (no instruction cost per byte);
// the dequantisation warps read them with conflict-free 16-byte shared
// loads.  Every role signals once per warp per stage, so the SM's issue
// slots go to the dequantisation arithmetic.  INT4 group scales are applied
// during dequantisation (bf16(q*s), one rounding); INT8 and FP8 per-channel
// scales are applied to the fp32 accumulator in the epilogue (exact
// factoring).
//
// Persistent CTAs (one per SM) walk the tile list (segment, 128-row weight
// block, BN-row token block) built on the device by the schedule kernel;
// one launch handles the experts of one weight format.  A CTA works on G
// tiles at a time (G = 2 for token blocks of up to 32 rows): K stage k of
// all G tiles forms one super-stage, produced, signalled and released as a
// unit, and each tile has its own MMA warp and accumulator, so one warp's
// barrier wait and commit overlap the other warp's MMAs -- a single issuing
// thread leaves the tensor pipe idle for several hundred cycles per stage,
// and every barrier operation costs a dequantisation warp ~200 cycles.
// Warp roles, all synchronised through mbarriers:
//   warp 0       : TMEM allocation; lane 0 streams raw weight tiles (bulk copy)
//   warp 1       : lane 0 issues the B tile loads (TMA)
//   warps 2, 3   : lane 0 of warp 2 + j issues the MMAs and commits of tile j
//   warps 4..11  : dequantise A into TMEM, as 2 groups of 4 warps that take
//                  alternate super-stages (so two are in flight); warp w
//                  owns TMEM lane quarter w % 4, one weight row per thread
//   warps 12..15 : epilogue (TMEM -> registers -> scales / SwiGLU -> bf16)
// Every wait is bounded: a role that waits ~1 s raises an abort flag, all
// roles drain what they issued, TMEM is freed and the error word is set.
#include <cuda.h>
#include <cuda_fp16.h>

#include <type_traits>

#include "qmoe_internal.cuh"

namespace qmoe {
namespace {

constexpr int kNDQ = 8;                        // dequantisation warps
constexpr int kGroups = kNDQ / 4;              // groups of 4 warps; group g converts super-stages g, g+2, ...
constexpr int kKW = kBK;                       // K elements one dequant thread converts per stage (its row)
constexpr int kHalf = kKW / 2;                 // converted and stored in two halves
constexpr int kRawWarp = 0, kBWarp = 1, kMmaWarp0 = 2;
constexpr int kMaxG = 2;                       // tiles in flight per CTA (one MMA warp each)
constexpr int kDQWarp0 = kMmaWarp0 + kMaxG;
constexpr int kEpiWarp0 = kDQWarp0 + kNDQ;
constexpr int kThreads = 32 * (kEpiWarp0 + 4);
constexpr int kTabMax = kMaxE + kMaxShared + 1;
constexpr uint32_t kTmemCols = 512;
// Poll back-off (ns) of the roles that wait off the critical path: the
// producers run ahead of the ring and the epilogue waits a whole tile.
constexpr uint32_t kSleepRaw = 128, kSleepB = 64, kSleepEpi = 256;

template <int FMT>
struct FmtCfg {
  static constexpr int SB = FMT == QMOE_W_INT4_G128 ? 128 * 64 + 256 : 128 * 128;  // bytes of a raw tile
  static constexpr int NC = FMT == QMOE_W_INT4_G128 ? kHalf / 32 : kHalf / 16;      // 16-byte chunks per half row
};

template <int BN, int FMT>
struct Cfg {
  static constexpr int G = BN <= 32 ? 2 : 1;                      // tiles in flight
  static constexpr int A_COL0 = 2 * G * BN;                       // TMEM: 2 accumulators per tile, then A
  static constexpr int SA0 = ((int)kTmemCols - A_COL0) / 64;
  static constexpr int SP = (SA0 > 7 ? 7 : SA0) / G;              // super-stage slots (G stages each)
  static constexpr int SA = SP * G;                               // A/B stage slots (TMEM + smem)
  static constexpr int B_STAGE = BN * 256;                        // BN rows x 128 K bf16
  static constexpr int STAGING = BN * 256;                        // epilogue staging
  static constexpr int SLOT = (FmtCfg<FMT>::SB + 127) & ~127;     // raw ring slot
  static constexpr int FIXED = SA * B_STAGE + STAGING + 6 * 1024;
  static constexpr int R0 = (224 * 1024 - FIXED) / SLOT;
  static constexpr int RP = (R0 > 16 ? 16 : R0) / G;              // raw ring: super-stage slots
  static constexpr int R = RP * G;                                // raw ring: tile slots
  static constexpr int OFF_B = 0;
  static constexpr int OFF_RAW = OFF_B + SA * B_STAGE;
  static constexpr int OFF_STG = OFF_RAW + R * SLOT;
  static constexpr int OFF_TAB = OFF_STG + STAGING;
  static constexpr int OFF_BAR = (OFF_TAB + 3 * kTabMax * 4 + 127) & ~127;
  static constexpr int NUM_BARS = 2 * SP + 2 * RP + 4 * G + G;
  static constexpr int OFF_MISC = (OFF_BAR + NUM_BARS * 8 + 15) & ~15;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;               // + alignment slack
  static_assert(RP >= 3 && SP >= 3, "rings too shallow");
  static_assert(G <= kMaxG, "MMA warps");
  static_assert(A_COL0 + SA * 64 <= (int)kTmemCols, "TMEM budget");
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(B_STAGE % 1024 == 0 && OFF_RAW % 1024 == 0 && OFF_BAR % 8 == 0 && OFF_MISC % 16 == 0,
                "alignment");
};

struct Tile {
  int seg, mb, row0, nvalid;
};

__device__ __forceinline__ Tile decode_tile(int tile, const int32_t* tab_off, const int32_t* seg_off,
                                            const int32_t* seg_cnt, int n_seg, int bn) {
  int lo = 0, hi = n_seg;  // largest seg with tab_off[seg] <= tile
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (tab_off[mid] <= tile) lo = mid; else hi = mid;
  }
  const int cnt = seg_cnt[lo];
  const int nblk = (cnt + bn - 1) / bn;
  const int local = tile - tab_off[lo];
  const int mb = local / nblk, nb = local - mb * nblk;
  Tile t;
  t.seg = lo;
  t.mb = mb;
  t.row0 = seg_off[lo] + nb * bn;
  t.nvalid = min(bn, cnt - nb * bn);
  return t;
}

// ---- dequantisation ----------------------------------------------------------
__device__ __forceinline__ uint32_t lop_and_or(uint32_t a, uint32_t mask, uint32_t orv) {
  return (a & mask) | orv;
}
__device__ __forceinline__ uint32_t bf2_sub(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t bf2_mul(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// 8 biased nibbles (q + 8) -> 4 bf16 pairs of q * s (one rounding).
__device__ __forceinline__ void deq_int4_word(uint32_t w, uint32_t s2, uint32_t* o) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t t = lop_and_or(w >> (4 * j), 0x000F000Fu, 0x43004300u);  // 128 + (q + 8)
    o[j] = bf2_mul(bf2_sub(t, 0x43084308u), s2);                           // (. - 136) * s
  }
}
// 4 int8 codes (byte order k0 k2 k1 k3) -> 2 bf16 pairs of q (exact).
__device__ __forceinline__ void deq_int8_word(uint32_t w, uint32_t* o) {
  o[0] = bf2_sub(lop_and_or(w, 0x007F007Fu, 0x43004300u), (w & 0x00800080u) ^ 0x43004300u);
  const uint32_t w8 = w >> 8;
  o[1] = bf2_sub(lop_and_or(w8, 0x007F007Fu, 0x43004300u), (w8 & 0x00800080u) ^ 0x43004300u);
}
// 4 e4m3 codes (byte order k0 k2 k1 k3) -> 2 bf16 pairs (exact): move the
// exponent/mantissa fields into bf16 position (value * 2^-120, subnormals
// included) and multiply by 2^120.
__device__ __forceinline__ void deq_fp8_word(uint32_t w, uint32_t* o) {
  const uint32_t lo = ((w << 4) & 0x07F007F0u) | ((w << 8) & 0x80008000u);
  const uint32_t hi = ((w >> 4) & 0x07F007F0u) | (w & 0x80008000u);
  o[0] = bf2_mul(lo, 0x7B807B80u);
  o[1] = bf2_mul(hi, 0x7B807B80u);
}

// 4 e4m3 codes (natural K order) -> 2 fp16 pairs (exact), one hardware
// conversion per pair of codes.
__device__ __forceinline__ void deq_fp8_f16_word(uint32_t w, uint32_t* o) {
  asm("{\n\t.reg .b16 lo, hi;\n\t"
      "mov.b32 {lo, hi}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, lo;\n\t"
      "cvt.rn.f16x2.e4m3x2 %1, hi;\n\t}"
      : "=r"(o[0]), "=r"(o[1])
      : "r"(w));
}

// This thread's 16-byte chunks (K order) -> kHalf / 2 bf16 (or fp16) pairs.
template <int FMT>
__device__ __forceinline__ void dequant_slice(const uint4 (&w)[FmtCfg<FMT>::NC], uint32_t sbits, uint32_t* av) {
#pragma unroll
  for (int c = 0; c < FmtCfg<FMT>::NC; ++c) {
    if constexpr (FMT == QMOE_W_INT4_G128) {
      const uint32_t s2 = sbits | (sbits << 16);
      deq_int4_word(w[c].x, s2, &av[16 * c + 0]);
      deq_int4_word(w[c].y, s2, &av[16 * c + 4]);
      deq_int4_word(w[c].z, s2, &av[16 * c + 8]);
      deq_int4_word(w[c].w, s2, &av[16 * c + 12]);
    } else if constexpr (FMT == kFmtFp8F16) {
      deq_fp8_f16_word(w[c].x, &av[8 * c + 0]);
      deq_fp8_f16_word(w[c].y, &av[8 * c + 2]);
      deq_fp8_f16_word(w[c].z, &av[8 * c + 4]);
      deq_fp8_f16_word(w[c].w, &av[8 * c + 6]);
    } else if constexpr (FMT == QMOE_W_FP8_E4M3_PC) {
      deq_fp8_word(w[c].x, &av[8 * c + 0]);
      deq_fp8_word(w[c].y, &av[8 * c + 2]);
      deq_fp8_word(w[c].z, &av[8 * c + 4]);
      deq_fp8_word(w[c].w, &av[8 * c + 6]);
    } else {
      deq_int8_word(w[c].x, &av[8 * c + 0]);
      deq_int8_word(w[c].y, &av[8 * c + 2]);
      deq_int8_word(w[c].z, &av[8 * c + 4]);
      deq_int8_word(w[c].w, &av[8 * c + 6]);
    }
  }
}

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + __expf(-g)); }

__device__ __forceinline__ uint16_t f2bf(float f) {
  const __nv_bfloat16 b = __float2bfloat16_rn(f);
  return *reinterpret_cast<const uint16_t*>(&b);
}
__device__ __forceinline__ uint16_t f2h(float f) {
  const __half h = __float2half_rn(f);
  return *reinterpret_cast<const uint16_t*>(&h);
}

// TMA: a box of 64 bf16 columns x BN rows of a row-major matrix into
// 128-byte-swizzled shared memory (rows past the matrix read as zero).
__device__ __forceinline__ void tma_tile2d(uint32_t dst, const CUtensorMap* map, int col, int row, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(col), "r"(row), "r"(smem_u32(bar))
      : "memory");
}

// Warp-uniform bounded wait: every lane polls, the warp proceeds together.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort));
}
// The same for roles off the critical path: back off between polls.
__device__ __forceinline__ bool warp_wait_backoff(uint64_t* bar, uint32_t parity, volatile int* abort, uint32_t ns) {
  return __all_sync(0xffffffffu, mbar_wait_backoff(bar, parity, abort, ns));
}

template <int BN, int MAT, int FMT>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const GemmArgs a, const __grid_constant__ CUtensorMap act_map) {
  using C = Cfg<BN, FMT>;
  using F = FmtCfg<FMT>;
  constexpr int G = C::G;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sB = smem + C::OFF_B;
  uint8_t* sRaw = smem + C::OFF_RAW;
  uint8_t* sStg = smem + C::OFF_STG;
  int32_t* tab_off = reinterpret_cast<int32_t*>(smem + C::OFF_TAB);
  int32_t* s_seg_off = tab_off + kTabMax;
  int32_t* s_seg_cnt = s_seg_off + kTabMax;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* full = bars;                      // [SP] B landed + A in TMEM, per super-stage
  uint64_t* empty = full + C::SP;             // [SP] MMAs done with the super-stage
  uint64_t* raw_full = empty + C::SP;         // [RP] raw tiles of a super-stage landed
  uint64_t* raw_empty = raw_full + C::RP;     // [RP] raw tiles consumed
  uint64_t* acc_full = raw_empty + C::RP;     // [G][2] accumulator of tile lane j, buffer b
  uint64_t* acc_empty = acc_full + 2 * G;     // [G][2]
  uint64_t* drain = acc_empty + 2 * G;        // [G]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_seg = a.n_seg;
  const int KS = a.K / kBK;

  if (tid == 0) {
    for (int s = 0; s < C::SP; ++s) {
      mbar_init(&full[s], 1 + 4);      // B producer expect_tx + one arrival per warp of a dequant group
      mbar_init(&empty[s], G);         // one commit per tile lane
    }
    for (int r = 0; r < C::RP; ++r) {
      mbar_init(&raw_full[r], 1);
      mbar_init(&raw_empty[r], 4);
    }
    for (int b = 0; b < 2 * G; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);     // one arrival per epilogue warp
    }
    for (int j = 0; j < G; ++j) mbar_init(&drain[j], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kRawWarp) tmem_alloc(tmem_slot, kTmemCols);
  // Everything above is private to the CTA and may overlap the previous
  // kernel's tail; the tile tables and the activations are read only after
  // that kernel has completed.
  pdl_wait();
  for (int i = tid; i <= n_seg; i += kThreads) {
    tab_off[i] = a.tile_off[i];
    if (i < n_seg) {
      s_seg_off[i] = a.seg_off[i];
      s_seg_cnt[i] = a.seg_cnt[i];
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = tab_off[n_seg];
  // This CTA's tiles: blockIdx.x + i * gridDim.x for i < nt, taken G at a
  // time.  A group of gq tiles is processed as KS super-stages; super-stage
  // ks holds K stage ks of every tile of the group (tile j in stage slot j of
  // the super-stage slot) and is produced, signalled and released as a unit.
  const int nt = (int)blockIdx.x < total ? (total - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;
  auto tile_of = [&](int i) { return decode_tile((int)blockIdx.x + i * (int)gridDim.x, tab_off, s_seg_off,
                                                 s_seg_cnt, n_seg, BN); };

  if (warp == kRawWarp) {
    // ---------------- raw weight tiles: one bulk copy per tile per K stage ----------------
    uint32_t rc = 0, r = 0, ph = 0;         // super-stages issued, ring slot, slot parity
    bool ok = true;
    for (int q0 = 0; q0 < nt && ok; q0 += G) {
      const int gq = min(G, nt - q0);
      const uint8_t* src[G];
#pragma unroll
      for (int j = 0; j < G; ++j) {
        if (j < gq) {
          const Tile t = tile_of(q0 + j);
          src[j] = a.experts[t.seg].w[MAT] + (size_t)t.mb * KS * F::SB;
        }
      }
      for (int ks = 0; ks < KS; ++ks) {
        ok = warp_wait_backoff(&raw_empty[r], ph ^ 1, abort_flag, kSleepRaw);
        if (!ok) break;
        if (lane == 0) {
          mbar_arrive_expect_tx(&raw_full[r], (uint32_t)(gq * F::SB));
#pragma unroll
          for (int j = 0; j < G; ++j)
            if (j < gq) bulk_g2s(sRaw + (r * G + j) * C::SLOT, src[j] + (size_t)ks * F::SB, F::SB, &raw_full[r]);
        }
        __syncwarp();
        ++rc;
        if (++r == (uint32_t)C::RP) { r = 0; ph ^= 1; }
      }
    }
    // wait for copies that may still be in flight before the CTA can exit
    if (lane == 0) {
      const uint32_t first = rc > (uint32_t)C::RP ? rc - C::RP : 0;
      for (uint32_t i = first; i < rc; ++i) mbar_wait_drain(&raw_full[i % C::RP], (i / C::RP) & 1);
    }
    __syncwarp();
  } else if (warp == kBWarp) {
    // ---------------- B rows: two TMA tiles per tile per K stage ----------------
    uint32_t sc = 0, s = 0, ph = 0;
    bool ok = true;
    for (int q0 = 0; q0 < nt && ok; q0 += G) {
      const int gq = min(G, nt - q0);
      int row0[G];
#pragma unroll
      for (int j = 0; j < G; ++j) row0[j] = j < gq ? tile_of(q0 + j).row0 : 0;
      for (int ks = 0; ks < KS; ++ks) {
        ok = warp_wait_backoff(&empty[s], ph ^ 1, abort_flag, kSleepB);
        if (!ok) break;
        if (lane == 0) {
          mbar_arrive_expect_tx(&full[s], (uint32_t)(gq * C::B_STAGE));
#pragma unroll
          for (int j = 0; j < G; ++j) {
            if (j < gq) {
              const uint32_t dst = smem_u32(sB + (s * G + j) * C::B_STAGE);
              tma_tile2d(dst, &act_map, ks * kBK, row0[j], &full[s]);
              tma_tile2d(dst + BN * 128, &act_map, ks * kBK + 64, row0[j], &full[s]);
            }
          }
        }
        __syncwarp();
        ++sc;
        if (++s == (uint32_t)C::SP) { s = 0; ph ^= 1; }
      }
    }
    if (lane == 0) {
      const uint32_t first = sc > (uint32_t)C::SP ? sc - C::SP : 0;
      for (uint32_t i = first; i < sc; ++i) mbar_wait_drain(&full[i % C::SP], (i / C::SP) & 1);
    }
    __syncwarp();
  } else if (warp < kDQWarp0) {
    // ---------------- MMA issuer of tile lane j (lane 0 alone) ----------------
    // A tight single-thread loop: the tensor pipe takes the next MMA only when
    // the previous one is nearly done, so any work between MMAs is exposed.
    const int j = warp - kMmaWarp0;
    if (j < G && lane == 0) {
      const uint64_t bdesc0 = smem_desc_sw128(smem_u32(sB + j * C::B_STAGE));
      const uint32_t a_tmem0 = tmem_base + C::A_COL0 + (uint32_t)(j * 64);
      bool ok = true;
      for (int q0 = 0, q = 0; q0 < nt && ok; q0 += G, ++q) {
        const int gq = min(G, nt - q0);
        if (j >= gq) break;
        const Tile t = tile_of(q0 + j);
        const int b = q & 1;
        ok = mbar_wait(&acc_empty[2 * j + b], ((q >> 1) & 1) ^ 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        const uint32_t idesc = idesc_bf16_m128(max(16, (t.nvalid + 15) & ~15), FMT == kFmtFp8F16);
        const uint32_t d_tmem = tmem_base + (uint32_t)((2 * j + b) * BN);
        const int u0 = q * KS;                 // super-stage index of this group's first K stage
        uint32_t s = (uint32_t)(u0 % C::SP), ph = (uint32_t)((u0 / C::SP) & 1);
        for (int ks = 0; ks < KS; ++ks) {
          if (!mbar_wait(&full[s], ph, abort_flag)) { ok = false; break; }
          tc_fence_after();
          // Descriptors of this stage: only the start-address field moves
          // (16-byte units), so each MMA's operands are one add away.
          const uint64_t bdesc = bdesc0 + (uint64_t)(s * (G * C::B_STAGE >> 4));
          const uint32_t a_tmem = a_tmem0 + s * (G * 64);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16_ts(d_tmem, a_tmem + kk * 8, bdesc + (uint64_t)((kk >> 2) * (BN * 128 >> 4) + (kk & 3) * 2),
                        idesc, (ks | kk) != 0);
          mma_commit(&empty[s]);
          for (int e = gq; e < G; ++e) mma_commit(&empty[s]);   // stand in for absent tile lanes
          if (++s == (uint32_t)C::SP) { s = 0; ph ^= 1; }
        }
        if (!ok) break;
        mma_commit(&acc_full[2 * j + b]);
      }
      if (!ok) {
        // let every MMA issued so far finish before TMEM is released
        mma_commit(&drain[j]);
        mbar_wait_drain(&drain[j], 0);
      }
    }
    __syncwarp();
  } else if (warp < kEpiWarp0) {
    // ---------------- A dequantisation into TMEM ----------------
    // Group g takes super-stages g, g + 2, g + 4, ...: it waits once for the
    // super-stage's raw tiles and its A slots, converts the gq tiles' K
    // stage (one weight row per thread, in two halves for register
    // pressure) into TMEM, and signals once.  A super-stage is published
    // (full barrier) only after the group's next one has been converted up
    // to its first store, so the store latency overlaps useful work.  This
    // cannot deadlock: that step waits only for the MMAs to release the slot
    // of super-stage u + 2 - SP, an earlier one (SP >= 3).
    const int q = warp & 3;                          // TMEM lane quarter
    const int g = (warp - kDQWarp0) >> 2;            // group
    const int row = 32 * q + lane;                   // weight row of the tile
    const uint32_t coff = (uint32_t)row * 16u;       // chunk-major raw tile
    const uint32_t soff = 128u * 64u + (uint32_t)row * 2u;   // INT4 group scale
    const uint32_t tbase = tmem_base + ((uint32_t)(32 * q) << 16) + C::A_COL0;
    const uint32_t raw0 = smem_u32(sRaw);
    constexpr int CPH = F::NC;                       // chunks per half row
    uint32_t s = 0, ph = 0, r = 0, rph = 0;          // ring positions of super-stage u
    int pending = -1;                                // A slot whose stores are not yet published
    bool ok = true;
    for (int q0 = 0, u = 0; q0 < nt && ok; q0 += G) {
      const int gq = min(G, nt - q0);
      for (int ks = 0; ks < KS; ++ks, ++u) {
        if (u % kGroups == g) {
          if (!(ok = warp_wait(&raw_full[r], rph, abort_flag))) break;
          for (int jj = 0; jj < gq; ++jj) {
            const uint32_t rp = raw0 + (r * G + jj) * C::SLOT;
            uint4 w0[CPH], w1[CPH];
#pragma unroll
            for (int k = 0; k < CPH; ++k) {
              asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                           : "=r"(w0[k].x), "=r"(w0[k].y), "=r"(w0[k].z), "=r"(w0[k].w)
                           : "r"(rp + coff + k * 2048));
              asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                           : "=r"(w1[k].x), "=r"(w1[k].y), "=r"(w1[k].z), "=r"(w1[k].w)
                           : "r"(rp + coff + (CPH + k) * 2048));
            }
            uint32_t sbits = 0;
            if constexpr (FMT == QMOE_W_INT4_G128) {
              unsigned short sv;
              asm volatile("ld.shared.u16 %0, [%1];" : "=h"(sv) : "r"(rp + soff));
              sbits = sv;
            }
            uint32_t av[kHalf / 2];
            dequant_slice<FMT>(w0, sbits, av);
            if (jj == 0) {
              if (!(ok = warp_wait(&empty[s], ph ^ 1, abort_flag))) break;
              tc_fence_after();               // TMEM stores after the MMAs' reads of this slot
              // The previous super-stage's stores were left in flight while
              // this one was loaded and converted; complete and publish them.
              if (pending >= 0) {
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&full[pending]);
              }
            }
            const uint32_t ta = tbase + (s * G + jj) * 64;
#pragma unroll
            for (int c = 0; c < kHalf / 32; ++c) tmem_st16(ta + 16 * c, &av[16 * c]);
            dequant_slice<FMT>(w1, sbits, av);
#pragma unroll
            for (int c = 0; c < kHalf / 32; ++c) tmem_st16(ta + kHalf / 2 + 16 * c, &av[16 * c]);
          }
          if (!ok) break;
          __syncwarp();
          if (lane == 0) mbar_arrive(&raw_empty[r]);
          pending = (int)s;
        }
        if (++r == (uint32_t)C::RP) { r = 0; rph ^= 1; }
        if (++s == (uint32_t)C::SP) { s = 0; ph ^= 1; }
      }
    }
    if (pending >= 0) {
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&full[pending]);
    }
  } else {
    // ---------------- epilogue ----------------
    // Each of the 4 epilogue warps owns 32 accumulator rows (TMEM lane
    // quarter q) and stages and stores its own slice of the output rows, so
    // only warp-level syncs are needed.  mat 0: 16 intermediate columns
    // (32 B) per token; mat 1: 32 output columns (64 B) per token.
    const int q = warp & 3;
    const int r = 32 * q + lane;             // accumulator row = tile weight row
    constexpr int WCOLS = MAT == 0 ? 16 : 32;
    uint16_t* stg = reinterpret_cast<uint16_t*>(sStg) + (size_t)q * BN * WCOLS;
    bool ok = true;
    for (int q0 = 0, grp = 0; q0 < nt && ok; q0 += G, ++grp) {
      const int gq = min(G, nt - q0);
      const int b = grp & 1;
      for (int j = 0; j < gq && ok; ++j) {
        const Tile t = tile_of(q0 + j);
        const ExpertDev& ex = a.experts[t.seg];
        const float scale = (FMT != QMOE_W_INT4_G128) ? ex.spc[MAT][t.mb * 128 + r] : 1.0f;
        ok = warp_wait_backoff(&acc_full[2 * j + b], (grp >> 1) & 1, abort_flag, kSleepEpi);
        if (!ok) break;
        tc_fence_after();
        const int n_mma = max(16, (t.nvalid + 15) & ~15);
        const uint32_t taddr = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)((2 * j + b) * BN);
        for (int c0 = 0; c0 < n_mma; c0 += 16) {
          uint32_t v[16];
          tmem_ld16(taddr + c0, v);
          tmem_wait_ld();
          if (MAT == 0) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float f = __uint_as_float(v[i]) * scale;
              const float o = __shfl_xor_sync(0xffffffffu, f, 1);   // up value of the same index
              if ((lane & 1) == 0) {
                const float hv = silu_f(f) * o;   // H is fp16 in the fp16 MMA mode, else bf16
                stg[(c0 + i) * WCOLS + (lane >> 1)] = FMT == kFmtFp8F16 ? f2h(hv) : f2bf(hv);
              }
            }
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) stg[(c0 + i) * WCOLS + lane] = f2bf(__uint_as_float(v[i]) * scale);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[2 * j + b]);
        constexpr int VPR = WCOLS / 8;         // 16-byte vectors per token row slice
        const int col0 = MAT == 0 ? t.mb * 64 + q * 16 : t.mb * 128 + q * 32;
        for (int v = lane; v < t.nvalid * VPR; v += 32) {
          const int n = v / VPR, c = v % VPR;
          *reinterpret_cast<uint4*>(a.out + (size_t)(t.row0 + n) * a.out_ld + col0 + c * 8) =
              *reinterpret_cast<const uint4*>(stg + n * WCOLS + c * 8);
        }
        __syncwarp();
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kRawWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
  if (tid == 0 && *abort_flag) atomicOr(a.err, kErrTimeout);
}

template <int BN, int MAT, int FMT>
cudaError_t launch_one(bool pdl, const GemmArgs& a, const CUtensorMap& map, int num_sms, cudaStream_t s) {
  using C = Cfg<BN, FMT>;
  auto kern = grouped_gemm_kernel<BN, MAT, FMT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  return launch_ex(kern, dim3(num_sms), dim3(kThreads), C::SMEM, s, pdl, a, map);
}

template <int BN, int MAT>
cudaError_t launch_fmt(bool pdl, const GemmArgs& a, const CUtensorMap& map, int fmt, int num_sms, cudaStream_t s) {
  switch (fmt) {
    case QMOE_W_INT4_G128: return launch_one<BN, MAT, QMOE_W_INT4_G128>(pdl, a, map, num_sms, s);
    case QMOE_W_FP8_E4M3_PC: return launch_one<BN, MAT, QMOE_W_FP8_E4M3_PC>(pdl, a, map, num_sms, s);
    case QMOE_W_INT8_PC: return launch_one<BN, MAT, QMOE_W_INT8_PC>(pdl, a, map, num_sms, s);
    case kFmtFp8F16: return launch_one<BN, MAT, kFmtFp8F16>(pdl, a, map, num_sms, s);
    default: return cudaErrorInvalidValue;
  }
}

template <int BN>
cudaError_t launch_bn(bool pdl, const GemmArgs& a, const CUtensorMap& map, int fmt, int num_sms, cudaStream_t s) {
  return a.mat == 0 ? launch_fmt<BN, 0>(pdl, a, map, fmt, num_sms, s) : launch_fmt<BN, 1>(pdl, a, map, fmt, num_sms, s);
}

}  // namespace

bool gemm_bn_supported(int bn) { return bn == 16 || bn == 32 || bn == 64 || bn == 128; }

cudaError_t launch_grouped_gemm(bool pdl, const GemmArgs& a, const CUtensorMap& act_map, int fmt, int bn, int num_sms,
                                cudaStream_t s) {
  switch (bn) {
    case 16: return launch_bn<16>(pdl, a, act_map, fmt, num_sms, s);
    case 32: return launch_bn<32>(pdl, a, act_map, fmt, num_sms, s);
    case 64: return launch_bn<64>(pdl, a, act_map, fmt, num_sms, s);
    case 128: return launch_bn<128>(pdl, a, act_map, fmt, num_sms, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace qmoe

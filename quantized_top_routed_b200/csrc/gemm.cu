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
//   D (M x N) = fp32 accumulators in tensor memory.
// Weights are the M side because an expert usually has few tokens: the
// weight stream is what the kernel moves.  Raw code tiles arrive by TMA bulk
// copy into a ring sized per weight format; the dequantisation warps read
// them with conflict-free 16-byte shared loads.  INT4 group scales are
// applied during dequantisation (bf16(q*s), one rounding); INT8 and FP8
// per-channel scales are applied to the fp32 accumulator in the epilogue
// (exact factoring).
//
// Issue rate.  One warp issues a tcgen05.mma about every 60-100 cycles
// whatever N is, while an M=128, N<=64, K=16 MMA needs far less tensor time;
// the rate grows with the number of warps issuing.  So the K stages of a
// tile are split into two classes (even and odd stage index), each with its
// own issuer warp accumulating into its own partial accumulator in TMEM; the
// epilogue adds the two partials in a fixed order (deterministic).
//
// Persistent CTAs (one per SM) walk the tile list (segment, 128-row weight
// block, BN-row token block) built on the device by the schedule kernel;
// one launch handles the experts of one weight format.  Each class has its
// own dequantisation group, issuer, partial (or D slots) and its own raw
// ring, A ring (TMEM) and B ring (shared memory), and each ring slot has a
// single producer warp.  So every ring slot has one producer and one
// consumer that both walk its uses in order, and a parity wait can never be
// two phases behind.
//
// Copy requests.  A TMA request holds the warp that issues it for several
// hundred cycles whatever its size (up to ~16 KB), while requests from
// different warps proceed in parallel.  So copies come from two producer
// warps, requests are large (the weight repack stores each class's stages
// of a block contiguously and one bulk copy brings NST of them; each K stage
// of B is one 3-D tensor box of 64 columns x BN rows x 2 column chunks), and
// the issuer warps issue nothing but MMAs.
//
// Per-stage scaling (INT4 group 128, BN <= 32).  A 128-K stage is one
// quantisation group, so A holds the exact codes q, each stage's MMAs write
// a D slot of their own, and the epilogue adds s(row, stage) * D into fp32
// registers in K order: the group scale is never rounded to bf16.
// Warp roles, all synchronised through mbarriers:
//   warps 0, 1   : producers (lane 0): raw weight chunks (bulk copies) and B
//                  stages (TMA) of class 0 / 1, or (BN >= 64) all raw
//                  chunks / all B stages; warp 0 also allocates TMEM
//   warps 2, 3   : MMA issuer of class 0 / 1 (warp-uniform loops, one
//                  elected lane issues)
//   warps 4..11  : dequantise A into TMEM, group c = warps 4 + 4c .. 7 + 4c;
//                  warp w owns TMEM lane quarter w % 4, one weight row per thread
//   warps 12..15 : epilogue (TMEM -> registers -> sum of partials, scales,
//                  SwiGLU -> bf16)
// Every wait is bounded (GemmArgs::wait_limit cycles): a role that waits too
// long raises an abort flag, all roles drain what they issued (copies on
// barriers that only their own bytes complete, MMAs on a commit), TMEM is
// freed and the error word is set.
#include <cuda.h>
#include <cuda_fp16.h>

#include "qmoe_internal.cuh"

namespace qmoe {
namespace {

constexpr int kProdWarp0 = 0, kMmaWarp0 = 2;  // producers: warps 0, 1
constexpr int kCls = 2;                        // stage classes (issuer warp + dequantisation group each)
constexpr int kDQWarp0 = kMmaWarp0 + kCls;     // first dequantisation warp
constexpr int kEpiWarp0 = kDQWarp0 + 4 * kCls;
constexpr int kThreads = 32 * (kEpiWarp0 + 4);
constexpr int kKW = kBK;                       // K elements one dequant thread converts per item (its row)
constexpr int kTabMax = kMaxE + kMaxShared + 1;
constexpr uint32_t kTmemCols = 512;
// Poll back-off (ns) of the roles that wait off the critical path: the
// producers run ahead of the rings and the epilogue waits a whole tile.
constexpr uint32_t kSleepRaw = 128, kSleepB = 64, kSleepEpi = 256;

template <int FMT>
struct FmtCfg {
  static constexpr int SB = FMT == QMOE_W_INT4_G128 ? 128 * 64 + 256 : 128 * 128;  // bytes of a raw tile
  static constexpr int QC = FMT == QMOE_W_INT4_G128 ? 1 : 2;    // 16-byte chunks per quarter row (16 pairs)
  static constexpr int NST = FMT == QMOE_W_INT4_G128 ? 2 : 1;   // stages per raw bulk copy (16.5 or 16 KB)
};

template <int BN, int FMT>
struct Cfg {
  // Per-stage scaling (INT4 group-128 with token blocks of up to 32 rows):
  // A holds the exact codes q, each class stage's MMAs write a D slot of
  // their own, and the epilogue adds s(row, stage) * D into fp32 registers.
  static constexpr bool PSS = FMT == QMOE_W_INT4_G128 && BN <= 32;
  static constexpr int NBUF = BN <= 32 ? 2 : 1;                      // accumulator sets (double buffer)
  static constexpr int DR = PSS ? (BN == 16 ? 4 : 2) : 0;            // D slots per class (per-stage mode)
  static constexpr int ACC = PSS ? kCls * DR * BN : NBUF * kCls * BN;   // TMEM columns of the accumulators
  static constexpr int SH0 = ((int)kTmemCols - ACC) / 64 / kCls;
  static constexpr int SH = SH0 > 3 ? 3 : SH0;                       // A slots (TMEM) per class
  static constexpr int SA = kCls * SH;
  // Producers: with wide token blocks (tensor-bound calls) one warp issues
  // the raw copies of both classes and the other the B boxes, so neither
  // kind of copy waits behind the other; with narrow ones each class has
  // its own producer warp issuing both.
  static constexpr bool SPLIT_PROD = BN >= 64;
  // Scale ring of the per-stage mode: slot i % SC of class c holds the fp32
  // scales of class item i.  SC >= SH + DR: the dequantisation of item
  // i + SC waits for the MMAs of item i + SC - SH, which waited for the D
  // slot that the epilogue freed after item i + SC - SH - DR >= i.
  static constexpr int SC = PSS ? SH + DR : 0;
  static constexpr int SCB = kCls * SC * 128 * 4;                    // bytes of the scale ring
  static constexpr int B_STAGE = BN * 256;                           // BN rows x 128 K bf16
  // B stages come from L2 with a TMA round trip of their own, so the B ring
  // runs deeper than the A ring (which TMEM bounds) where shared memory allows.
  static constexpr int SHB0 = 96 * 1024 / B_STAGE / kCls;
  static constexpr int SHB = SHB0 > 8 ? 8 : (SHB0 < 2 ? 2 : SHB0);   // B slots per class
  static constexpr int SB = kCls * SHB;
  static constexpr int STAGING = 4 * 16 * (BN <= 32 ? BN / 16 : 1) * 64;   // epilogue staging (4 warps)
  static constexpr int NST = FmtCfg<FMT>::NST;
  static constexpr int CHUNK = NST * FmtCfg<FMT>::SB;                // raw ring slot
  static constexpr int FIXED = SB * B_STAGE + STAGING + SCB + 6 * 1024;
  static constexpr int R0 = (224 * 1024 - FIXED) / CHUNK / kCls;
  static constexpr int RH = R0 > 8 ? 8 : R0;                         // raw slots per class
  static constexpr int R = kCls * RH;
  static constexpr int OFF_B = 0;
  static constexpr int OFF_RAW = OFF_B + SB * B_STAGE;
  static constexpr int OFF_STG = OFF_RAW + R * CHUNK;
  static constexpr int OFF_SC = (OFF_STG + STAGING + 127) & ~127;
  static constexpr int OFF_TAB = (OFF_SC + SCB + 127) & ~127;
  static constexpr int OFF_BAR = (OFF_TAB + 3 * kTabMax * 4 + 127) & ~127;
  static constexpr int NUM_BARS = 2 * SA + 2 * SB + 2 * R + 2 * NBUF + kCls + (PSS ? 2 * kCls * DR + kCls * SC : 0);
  static constexpr int OFF_MISC = (OFF_BAR + NUM_BARS * 8 + 15) & ~15;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;                  // + alignment slack
  static_assert(RH >= 2 && SH >= 2, "rings too shallow");
  static_assert(ACC + SA * 64 <= (int)kTmemCols, "TMEM budget");
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(B_STAGE % 1024 == 0 && OFF_RAW % 1024 == 0 && CHUNK % 16 == 0 && OFF_BAR % 8 == 0 &&
                    OFF_MISC % 16 == 0,
                "alignment");
};

struct Tile {
  int seg, mb, row0, nvalid;
};

__device__ __forceinline__ Tile decode_tile(int tile, const int32_t* tab_off, const int32_t* seg_off,
                                            const int32_t* seg_cnt, int n_seg, int bn, int group) {
  int lo = 0, hi = n_seg;  // largest seg with tab_off[seg] <= tile
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (tab_off[mid] <= tile) lo = mid; else hi = mid;
  }
  const int cnt = seg_cnt[lo];
  const int nblk = (cnt + bn - 1) / bn;
  const int local = tile - tab_off[lo];
  int mb, nb;
  if (group > 0 && nblk > group) {
    // groups of `group` token blocks; inside a group, weight block major
    const int nmb = (tab_off[lo + 1] - tab_off[lo]) / nblk;
    const int per = nmb * group;
    const int g = local / per;
    const int gsz = min(group, nblk - g * group);
    const int rem = local - g * per;
    mb = rem / gsz;
    nb = g * group + rem % gsz;
  } else {
    mb = local / nblk;
    nb = local - mb * nblk;
  }
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
// 8 biased nibbles (q + 8) -> 4 bf16 pairs of q (exact; the group scale is
// applied to the stage's fp32 result instead).
__device__ __forceinline__ void deq_int4_word_q(uint32_t w, uint32_t* o) {
#pragma unroll
  for (int j = 0; j < 4; ++j)
    o[j] = bf2_sub(lop_and_or(w >> (4 * j), 0x000F000Fu, 0x43004300u), 0x43084308u);   // 136 + q - 136
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

// NCHK of this thread's 16-byte chunks (K order) -> bf16 (or fp16) pairs.
template <int FMT, int NCHK, bool PSS = false>
__device__ __forceinline__ void dequant_chunks(const uint4* w, uint32_t sbits, uint32_t* av) {
#pragma unroll
  for (int c = 0; c < NCHK; ++c) {
    if constexpr (PSS) {
      deq_int4_word_q(w[c].x, &av[16 * c + 0]);
      deq_int4_word_q(w[c].y, &av[16 * c + 4]);
      deq_int4_word_q(w[c].z, &av[16 * c + 8]);
      deq_int4_word_q(w[c].w, &av[16 * c + 12]);
    } else if constexpr (FMT == QMOE_W_INT4_G128) {
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

// silu(g) * u with the fast exponential and division: the layer's output
// tolerance is far above their few-ulp error.
__device__ __forceinline__ float swiglu_f(float g, float u) { return __fdividef(g, 1.0f + __expf(-g)) * u; }

__device__ __forceinline__ uint16_t f2bf(float f) {
  const __nv_bfloat16 b = __float2bfloat16_rn(f);
  return *reinterpret_cast<const uint16_t*>(&b);
}
__device__ __forceinline__ uint16_t f2h(float f) {
  const __half h = __float2half_rn(f);
  return *reinterpret_cast<const uint16_t*>(&h);
}

// TMA: a 3-D box (64 columns x BN rows x 2 column chunks = one K stage of B)
// of a row-major matrix viewed as (64, rows, cols / 64) into 128-byte-swizzled
// shared memory laid out [chunk][row][64] (rows past the matrix read as zero).
__device__ __forceinline__ void tma_tile3d(uint32_t dst, const CUtensorMap* map, int x, int y, int z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

// Warp-uniform bounded wait: every lane polls, the warp proceeds together.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, long long lim) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, lim));
}
// The same for roles off the critical path: back off between polls.
__device__ __forceinline__ bool warp_wait_backoff(uint64_t* bar, uint32_t parity, volatile int* abort, uint32_t ns,
                                                  long long lim) {
  return __all_sync(0xffffffffu, mbar_wait_backoff(bar, parity, abort, ns, lim));
}

template <int BN, int MAT, int FMT>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const GemmArgs a, const __grid_constant__ CUtensorMap act_map) {
  using C = Cfg<BN, FMT>;
  using F = FmtCfg<FMT>;
  constexpr int SH = C::SH, SHB = C::SHB, RH = C::RH, NBUF = C::NBUF, NST = C::NST;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sB = smem + C::OFF_B;
  uint8_t* sRaw = smem + C::OFF_RAW;
  uint8_t* sStg = smem + C::OFF_STG;
  int32_t* tab_off = reinterpret_cast<int32_t*>(smem + C::OFF_TAB);
  int32_t* s_seg_off = tab_off + kTabMax;
  int32_t* s_seg_cnt = s_seg_off + kTabMax;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* full = bars;                      // [SA] A of the item in TMEM (one arrival per dequant warp)
  uint64_t* empty = full + C::SA;             // [SA] MMAs done with the A slot
  uint64_t* bfull = empty + C::SA;            // [SB] B stage of the item landed (TMA bytes only)
  uint64_t* bempty = bfull + C::SB;           // [SB] MMAs done with the B slot
  uint64_t* raw_full = bempty + C::SB;        // [R] raw tile of the item landed
  uint64_t* raw_empty = raw_full + C::R;      // [R] raw tile consumed
  uint64_t* acc_full = raw_empty + C::R;      // [NBUF] both partials of the tile complete
  uint64_t* acc_empty = acc_full + NBUF;      // [NBUF] the epilogue has read the partials
  uint64_t* drain = acc_empty + NBUF;         // [kCls] abort path of the issuers
  uint64_t* dfull = drain + kCls;             // [kCls * DR] per-stage mode: the stage's D slot is complete
  uint64_t* dempty = dfull + kCls * C::DR;    // [kCls * DR] per-stage mode: the epilogue has read the D slot
  uint64_t* scfull = dempty + kCls * C::DR;   // [kCls * SC] per-stage mode: the item's scales are written
  float* sScale = reinterpret_cast<float*>(smem + C::OFF_SC);   // [kCls][SC][128]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_seg = a.n_seg;
  const int KS = a.K / kBK;
  const long long lim = a.wait_limit;
  // Items of a class: stage ks of the CTA's tile q with ks = c (mod 2) is
  // class stage j = ks / 2 of the tile and has class index i = q * ncls(c) + j;
  // it uses A slot c * SH + i % SH and B slot c * SHB + i % SHB.  Its raw
  // codes arrive in chunk g = q * nchunk(c) + j / NST (NST consecutive class
  // stages, one bulk copy), raw slot c * RH + g % RH.
  auto ncls = [&](int c) { return (KS + 1 - c) >> 1; };
  auto nchunk = [&](int c) { return (ncls(c) + NST - 1) / NST; };

  if (tid == 0) {
    for (int s = 0; s < C::SA; ++s) {
      mbar_init(&full[s], 4);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < C::SB; ++s) {
      mbar_init(&bfull[s], 1);
      mbar_init(&bempty[s], 1);
    }
    for (int r = 0; r < C::R; ++r) {
      mbar_init(&raw_full[r], 1);
      mbar_init(&raw_empty[r], 4);
    }
    for (int b = 0; b < NBUF; ++b) {
      mbar_init(&acc_full[b], kCls);   // one arrival per issuer
      mbar_init(&acc_empty[b], 4);     // one arrival per epilogue warp
    }
    for (int c = 0; c < kCls; ++c) mbar_init(&drain[c], 1);
    for (int d = 0; d < kCls * C::DR; ++d) {
      mbar_init(&dfull[d], 1);
      mbar_init(&dempty[d], 4);        // one arrival per epilogue warp
    }
    for (int d = 0; d < kCls * C::SC; ++d) mbar_init(&scfull[d], 4);   // one arrival per dequant warp
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kProdWarp0) tmem_alloc(tmem_slot, kTmemCols);
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
#ifdef QMOE_DEBUG
  // The tile tables come from data (the schedule's output): check them
  // before any role uses them, and give every role of the CTA no tiles if
  // they are bad, so all roles stay consistent.
  volatile int* tab_bad = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);
  if (tid == 0) {
    int bad = tab_off[0] != 0;
    for (int i = 0; i < n_seg && !bad; ++i) {
      const int cnt = s_seg_cnt[i], tiles = tab_off[i + 1] - tab_off[i];
      const int want = ((cnt + BN - 1) / BN) * a.MB;
      bad = cnt < 0 || s_seg_off[i] < 0 || s_seg_off[i] + cnt > a.rows || (tiles != 0 && tiles != want);
    }
    *tab_bad = bad;
  }
  __syncthreads();
  const bool tab_ok = dbg_in_bounds(*tab_bad == 0, tid == 0 ? a.err : nullptr);
#else
  constexpr bool tab_ok = true;
#endif
  const int total = tab_ok ? tab_off[n_seg] : 0;
  // This CTA's tiles: blockIdx.x + q * gridDim.x for q < nt.
  const int nt = (int)blockIdx.x < total ? (total - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;
  // Down GEMM: the token blocks of an expert are visited in groups of 8, and
  // inside a group weight block major, so a group's H rows stay in L2 while
  // all weight blocks pass over them.  (Gate/up keeps weight block major over
  // all token blocks: its x rows are small next to W13.)
  constexpr int kGroup = MAT == 1 ? 8 : 0;
  auto tile_of = [&](int q) { return decode_tile((int)blockIdx.x + q * (int)gridDim.x, tab_off, s_seg_off,
                                                 s_seg_cnt, n_seg, BN, kGroup); };

  if (warp < kMmaWarp0) {
    // ---------------- producer of class c: raw chunks and B stages ----------------
    // Items in order: the raw chunk when an item starts one (NST class stages
    // per bulk copy), then the item's B stage (one 3-D tensor box).
    if constexpr (C::SPLIT_PROD) {
    // warp 0: raw chunks of both classes; warp 1: B stages of both classes
    bool ok = true;
    uint32_t issued[kCls] = {0, 0};
    if (warp == kProdWarp0) {
      for (int q = 0; q < nt && ok; ++q) {
        const Tile t = tile_of(q);
        const uint8_t* base = a.experts[t.seg].w[MAT] + (size_t)t.mb * KS * F::SB;
        for (int m = 0; m < nchunk(0) && ok; ++m) {
          for (int c = 0; c < kCls; ++c) {
            const int nc = ncls(c), nch = nchunk(c);
            if (m >= nch) continue;
            const uint32_t g = (uint32_t)(q * nch + m);
            const uint32_t r = c * RH + g % RH, ph = (g / RH) & 1;
            if (!(ok = warp_wait_backoff(&raw_empty[r], ph ^ 1, abort_flag, kSleepRaw, lim))) break;
            const uint32_t bytes = (uint32_t)(min(NST, nc - m * NST) * F::SB);
            const size_t pos = (size_t)(c ? ncls(0) : 0) + (size_t)m * NST;
            if (lane == 0) {
              mbar_arrive_expect_tx(&raw_full[r], bytes);
              bulk_g2s(sRaw + r * C::CHUNK, base + pos * F::SB, bytes, &raw_full[r]);
            }
            __syncwarp();
            issued[c] = g + 1;
          }
        }
      }
      if (lane == 0)
        for (int c = 0; c < kCls; ++c) {
          const uint32_t first = issued[c] > (uint32_t)RH ? issued[c] - RH : 0;
          for (uint32_t g = first; g < issued[c]; ++g) mbar_wait_drain(&raw_full[c * RH + g % RH], (g / RH) & 1);
        }
    } else {
      for (int q = 0; q < nt && ok; ++q) {
        const Tile t = tile_of(q);
        for (int ks = 0; ks < KS; ++ks) {
          const int c = ks & 1, j = ks >> 1;
          const uint32_t i = (uint32_t)(q * ncls(c) + j);
          const uint32_t sb = c * SHB + i % SHB, pb = (i / SHB) & 1;
          if (!(ok = warp_wait_backoff(&bempty[sb], pb ^ 1, abort_flag, kSleepB, lim))) break;
          if (lane == 0) {
            mbar_arrive_expect_tx(&bfull[sb], (uint32_t)C::B_STAGE);
            tma_tile3d(smem_u32(sB + sb * C::B_STAGE), &act_map, 0, t.row0, 2 * ks, &bfull[sb]);
          }
          __syncwarp();
          issued[c] = i + 1;
        }
      }
      if (lane == 0)
        for (int c = 0; c < kCls; ++c) {
          const uint32_t first = issued[c] > (uint32_t)SHB ? issued[c] - SHB : 0;
          for (uint32_t i = first; i < issued[c]; ++i) mbar_wait_drain(&bfull[c * SHB + i % SHB], (i / SHB) & 1);
        }
    }
    __syncwarp();
    } else {
    const int c = warp - kProdWarp0;
    const int nc = ncls(c), nch = nchunk(c);
    const int first_pos = c ? ncls(0) : 0;   // position of the class's first stage in a block
    bool ok = true;
    uint32_t raw_issued = 0, b_issued = 0;
    for (int q = 0; q < nt && ok; ++q) {
      const Tile t = tile_of(q);
      const uint8_t* src = a.experts[t.seg].w[MAT] + ((size_t)t.mb * KS + first_pos) * F::SB;
      for (int j = 0; j < nc; ++j) {
        if (j % NST == 0) {
          const int m = j / NST;
          const uint32_t g = (uint32_t)(q * nch + m);
          const uint32_t r = c * RH + g % RH, ph = (g / RH) & 1;
          if (!(ok = warp_wait_backoff(&raw_empty[r], ph ^ 1, abort_flag, kSleepRaw, lim))) break;
          const uint32_t bytes = (uint32_t)(min(NST, nc - m * NST) * F::SB);
          if (lane == 0) {
            mbar_arrive_expect_tx(&raw_full[r], bytes);
            bulk_g2s(sRaw + r * C::CHUNK, src + (size_t)m * NST * F::SB, bytes, &raw_full[r]);
          }
          __syncwarp();
          raw_issued = g + 1;
        }
        const uint32_t i = (uint32_t)(q * nc + j);
        const uint32_t sb = c * SHB + i % SHB, pb = (i / SHB) & 1;
        if (!(ok = warp_wait_backoff(&bempty[sb], pb ^ 1, abort_flag, kSleepB, lim))) break;
        if (lane == 0) {
          mbar_arrive_expect_tx(&bfull[sb], (uint32_t)C::B_STAGE);
          tma_tile3d(smem_u32(sB + sb * C::B_STAGE), &act_map, 0, t.row0, 2 * (2 * j + c), &bfull[sb]);
        }
        __syncwarp();
        b_issued = i + 1;
      }
    }
    // copies that may still be in flight land before the CTA can exit (each
    // barrier completes on its own copies' bytes alone)
    if (lane == 0) {
      const uint32_t first = raw_issued > (uint32_t)RH ? raw_issued - RH : 0;
      for (uint32_t g = first; g < raw_issued; ++g) mbar_wait_drain(&raw_full[c * RH + g % RH], (g / RH) & 1);
      const uint32_t firstb = b_issued > (uint32_t)SHB ? b_issued - SHB : 0;
      for (uint32_t i = firstb; i < b_issued; ++i) mbar_wait_drain(&bfull[c * SHB + i % SHB], (i / SHB) & 1);
    }
    __syncwarp();
    }
  } else if (warp < kDQWarp0) {
    // ---------------- MMA issuer of class c ----------------
    // Class stages ks = c, c + 2, ... of every tile, accumulated into partial
    // c of the tile's accumulator set (per-stage mode: each stage into the
    // next D slot of the class).  The loop runs on the whole warp; one
    // elected lane issues.
    const int c = warp - kMmaWarp0;
    const uint64_t bdesc0 = smem_desc_sw128(smem_u32(sB));
    const uint32_t a_tmem0 = tmem_base + C::ACC;
    const int nc = ncls(c);
    bool ok = true;
    for (int q = 0; q < nt && ok; ++q) {
      const Tile t = tile_of(q);
      const uint32_t idesc = idesc_bf16_m128(max(16, (t.nvalid + 15) & ~15), FMT == kFmtFp8F16);
      const int b = NBUF == 2 ? (q & 1) : 0;    // accumulator set of this tile
      const int use = NBUF == 2 ? (q >> 1) : q;  // its use count before this tile
      // the epilogue has read this set's previous tile
      if (!C::PSS && !(ok = warp_wait(&acc_empty[b], (use & 1) ^ 1, abort_flag, lim))) break;
      uint32_t d_tmem = tmem_base + (uint32_t)((b * kCls + c) * BN);
      for (int j = 0; j < nc; ++j) {
        const uint32_t i = (uint32_t)(q * nc + j);
        const uint32_t s = c * SH + i % SH, ph = (i / SH) & 1;
        const uint32_t sb = c * SHB + i % SHB, pb = (i / SHB) & 1;
        const uint32_t ds = c * C::DR + (C::PSS ? i % C::DR : 0);
        if constexpr (C::PSS) {                  // the epilogue has read this D slot's previous stage
          if (!(ok = warp_wait(&dempty[ds], ((i / C::DR) & 1) ^ 1, abort_flag, lim))) break;
          d_tmem = tmem_base + ds * BN;
        }
        if (!(ok = warp_wait(&bfull[sb], pb, abort_flag, lim))) break;
        if (!(ok = warp_wait(&full[s], ph, abort_flag, lim))) break;
        tc_fence_after();
        // Descriptors of these slots: only the start-address field moves
        // (16-byte units), so each MMA's operands are one add away.
        const uint64_t bdesc = bdesc0 + (uint64_t)(sb * (C::B_STAGE >> 4));
        const uint32_t a_tmem = a_tmem0 + s * 64;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ts_elect(d_tmem, a_tmem + kk * 8,
                            bdesc + (uint64_t)((kk >> 2) * (BN * 128 >> 4) + (kk & 3) * 2), idesc,
                            ((C::PSS ? 0 : j) != 0 || kk != 0) ? 1u : 0u);
        mma_commit_elect(&empty[s]);
        mma_commit_elect(&bempty[sb]);
        if constexpr (C::PSS) mma_commit_elect(&dfull[ds]);
      }
      if (!ok) break;
      if constexpr (C::PSS) continue;
      if (nc > 0) {
        mma_commit_elect(&acc_full[b]);
      } else {                                 // a one-stage K: class 1 has nothing to add
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_full[b]);
      }
    }
    // Every MMA this warp issued completes before TMEM is released: after an
    // abort the epilogue may not have waited for the last ones.
    mma_commit_elect(&drain[c]);
    mbar_wait_drain(&drain[c], 0);
    __syncwarp();
  } else if (warp < kEpiWarp0) {
    // ---------------- A dequantisation into TMEM ----------------
    // Group c converts the class-c items in order: it loads its row of the
    // stage's raw codes, converts the first quarter, waits for the A slot,
    // stores it, converts and stores the other quarters, and signals the item
    // (and frees the raw chunk after its last stage).
    const int q = warp & 3;                          // TMEM lane quarter
    const int c = (warp - kDQWarp0) >> 2;            // class
    const int row = 32 * q + lane;                   // weight row of the tile
    const uint32_t coff = (uint32_t)row * 16u;       // chunk-major raw tile
    const uint32_t soff = 128u * 64u + (uint32_t)row * 2u;   // INT4 group scale
    const uint32_t tbase = tmem_base + ((uint32_t)(32 * q) << 16) + C::ACC;
    const uint32_t raw0 = smem_u32(sRaw);
    constexpr int QC = F::QC;
    const int nc = ncls(c), nch = nchunk(c);
    bool ok = true;
    for (int tq = 0; tq < nt && ok; ++tq) {
     for (int j = 0; j < nc; ++j) {
      const uint32_t i = (uint32_t)(tq * nc + j);
      const int m = j / NST, kin = j - m * NST;     // chunk of the class stage and position in it
      const uint32_t g = (uint32_t)(tq * nch + m);
      const uint32_t r = c * RH + g % RH, rph = (g / RH) & 1;
      const uint32_t s = c * SH + i % SH, ph = (i / SH) & 1;
      if (!(ok = warp_wait(&raw_full[r], rph, abort_flag, lim))) break;
      const uint32_t rp = raw0 + r * C::CHUNK + kin * F::SB;
      uint4 w[4 * QC];                           // the row's 128 K of codes
#pragma unroll
      for (int k = 0; k < 4 * QC; ++k)
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(w[k].x), "=r"(w[k].y), "=r"(w[k].z), "=r"(w[k].w)
                     : "r"(rp + coff + k * 2048));
      uint32_t sbits = 0;
      if constexpr (FMT == QMOE_W_INT4_G128) {
        unsigned short sv;
        asm volatile("ld.shared.u16 %0, [%1];" : "=h"(sv) : "r"(rp + soff));
        sbits = sv;
      }
      // Four quarters of 16 pairs, converted into two alternating register
      // sets so a conversion never waits for the previous quarter's store to
      // read its registers.
      uint32_t av[2][16];
      dequant_chunks<FMT, QC, C::PSS>(&w[0], sbits, av[0]);
      if (!(ok = warp_wait(&empty[s], ph ^ 1, abort_flag, lim))) break;
      tc_fence_after();                          // TMEM stores after the MMAs' reads of this slot
      const uint32_t ta = tbase + s * 64;
      tmem_st16(ta, av[0]);
      const uint32_t scs = (uint32_t)c * C::SC + (C::PSS ? i % C::SC : 0);   // scale slot (per-stage mode)
      if constexpr (C::PSS) sScale[scs * 128 + row] = __uint_as_float(sbits << 16);
#pragma unroll
      for (int qq = 1; qq < 4; ++qq) {
        dequant_chunks<FMT, QC, C::PSS>(&w[qq * QC], sbits, av[qq & 1]);
        tmem_st16(ta + 16 * qq, av[qq & 1]);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (C::PSS) mbar_arrive(&scfull[scs]);
        mbar_arrive(&full[s]);
        if (kin == NST - 1 || j == nc - 1) mbar_arrive(&raw_empty[r]);   // last stage of the chunk
      }
     }
    }
    if (!ok) tmem_wait_st();                         // stores issued before the abort land first
  } else {
    // ---------------- epilogue ----------------
    // Each of the 4 epilogue warps owns 32 accumulator rows (TMEM lane
    // quarter q), adds the tile's two partials (class 0 + class 1), and
    // stages and stores its own slice of the output rows, so only warp-level
    // syncs are needed.  mat 0: 16 intermediate columns (32 B) per token;
    // mat 1: 32 output columns (64 B) per token.
    const int q = warp & 3;
    const int r = 32 * q + lane;             // accumulator row = tile weight row
    constexpr int WCOLS = MAT == 0 ? 16 : 32;
    constexpr int NCH = BN <= 32 ? BN / 16 : 1;   // 16-column chunks held in registers at once
    uint16_t* stg = reinterpret_cast<uint16_t*>(sStg) + (size_t)q * 16 * NCH * WCOLS;   // [16 * NCH tokens][WCOLS]
    const bool two = KS > 1;                 // class 1 received K stages
    bool ok = true;
    // Output of columns [c0, c0 + 16 * NCH) of the tile (v: the fp32
    // accumulator row of this thread for those token columns).
    auto emit = [&](const Tile& t, int c0, int n_mma, float (&v)[NCH][16]) {
#pragma unroll
      for (int ch = 0; ch < NCH; ++ch) {
        const int cc = c0 + 16 * ch;
        if (cc >= n_mma) break;
        if (MAT == 0) {
          // Lanes 2i (gate row) and 2i+1 (up row) share the SwiGLU of
          // intermediate index i: the even lane produces columns 0-7 of the
          // chunk, the odd lane columns 8-15.
          const bool odd = lane & 1;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float send = odd ? v[ch][i] : v[ch][i + 8];
            const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
            const float hv = odd ? swiglu_f(recv, v[ch][i + 8]) : swiglu_f(v[ch][i], recv);
            const int col = 16 * ch + i + (odd ? 8 : 0);
            // H is fp16 in the fp16 MMA mode, else bf16
            stg[col * WCOLS + (lane >> 1)] = FMT == kFmtFp8F16 ? f2h(hv) : f2bf(hv);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) stg[(16 * ch + i) * WCOLS + lane] = f2bf(v[ch][i]);
        }
      }
      // this warp's slice of the staged tokens, coalesced 16-byte stores
      __syncwarp();
      constexpr int VPR = WCOLS / 8;       // 16-byte vectors per token row slice
      const int col0 = MAT == 0 ? t.mb * 64 + q * 16 : t.mb * 128 + q * 32;
      const int nrows = min(16 * NCH, t.nvalid - c0);
      for (int u = lane; u < nrows * VPR; u += 32) {
        const int n = u / VPR, cv = u % VPR;
        *reinterpret_cast<uint4*>(a.out + (size_t)(t.row0 + c0 + n) * a.out_ld + col0 + cv * 8) =
            *reinterpret_cast<const uint4*>(stg + n * WCOLS + cv * 8);
      }
      __syncwarp();
    };
    for (int tq = 0; tq < nt && ok; ++tq) {
      const Tile t = tile_of(tq);
      const int n_mma = max(16, (t.nvalid + 15) & ~15);
      if constexpr (C::PSS) {
        // Stages in K order (the classes alternate): acc += s(row, stage) * D.
        float v[NCH][16];
#pragma unroll
        for (int ch = 0; ch < NCH; ++ch)
#pragma unroll
          for (int i = 0; i < 16; ++i) v[ch][i] = 0.f;
        for (int ks = 0; ks < KS; ++ks) {
          const int c = ks & 1;
          const uint32_t i = (uint32_t)(tq * ncls(c) + (ks >> 1));
          const uint32_t ds = c * C::DR + i % C::DR, scs = c * C::SC + i % C::SC;
          if (!(ok = warp_wait(&dfull[ds], (i / C::DR) & 1, abort_flag, lim))) break;
          if (!(ok = warp_wait(&scfull[scs], (i / C::SC) & 1, abort_flag, lim))) break;
          tc_fence_after();
          const float sc = sScale[scs * 128 + r];
          const uint32_t taddr = tmem_base + ((uint32_t)(32 * q) << 16) + ds * BN;
          uint32_t x[NCH][16];
#pragma unroll
          for (int ch = 0; ch < NCH; ++ch)
            if (16 * ch < n_mma) tmem_ld16(taddr + 16 * ch, x[ch]);
          tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&dempty[ds]);   // the scale was read above, before the release
#pragma unroll
          for (int ch = 0; ch < NCH; ++ch)
            if (16 * ch < n_mma) {
#pragma unroll
              for (int e = 0; e < 16; ++e) v[ch][e] = fmaf(sc, __uint_as_float(x[ch][e]), v[ch][e]);
            }
        }
        if (!ok) break;
        emit(t, 0, n_mma, v);
      } else {
        const ExpertDev& ex = a.experts[t.seg];
        const float scale = (FMT != QMOE_W_INT4_G128) ? ex.spc[MAT][t.mb * 128 + r] : 1.0f;
        const int b = NBUF == 2 ? (tq & 1) : 0;
        const int use = NBUF == 2 ? (tq >> 1) : tq;
        ok = warp_wait_backoff(&acc_full[b], use & 1, abort_flag, kSleepEpi, lim);
        if (!ok) break;
        tc_fence_after();
        const uint32_t taddr = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(b * kCls * BN);
        // Columns [c0, c0 + 16 * NCH) of partial 0 + partial 1, then the output
        // for them.  For token blocks of up to 32 rows every column is read
        // before the set is released, so the issuers can start the tile after
        // next while this one is finished.
        for (int c0 = 0; c0 < n_mma; c0 += 16 * NCH) {
          float v[NCH][16];
#pragma unroll
          for (int ch = 0; ch < NCH; ++ch) {
            if (c0 + 16 * ch < n_mma) {
              const uint32_t col = taddr + c0 + 16 * ch;
              uint32_t x0[16], x1[16];
              tmem_ld16(col, x0);
              if (two) tmem_ld16(col + BN, x1);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 16; ++i)
                v[ch][i] = (two ? __uint_as_float(x0[i]) + __uint_as_float(x1[i]) : __uint_as_float(x0[i])) * scale;
            }
          }
          if (c0 + 16 * NCH >= n_mma) {             // last columns read: release the set
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[b]);
          }
          emit(t, c0, n_mma, v);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kProdWarp0) {
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

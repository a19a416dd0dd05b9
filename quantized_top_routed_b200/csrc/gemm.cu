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
//   B (N x K) = up to BN rows of the expert's segment (tokens), gathered
//               from x / H into 128-byte-swizzled shared memory (cp.async);
//   D (M x N) = fp32 accumulators in tensor memory, double buffered.
// Weights are the M side because an expert usually has few tokens; the
// weight stream is what the kernel moves.  INT4 group scales are applied
// during dequantisation (bf16(q*s), one rounding); INT8 and FP8 per-channel
// scales are applied to the fp32 accumulator in the epilogue (exact
// factoring).
//
// Persistent CTAs (one per SM) walk the tile list (segment, 128-row weight
// block, BN-row token block) built on the device by the schedule kernel.
// Warp roles, all synchronised through mbarriers:
//   warp 0      : TMEM allocation; lane 0 streams raw weight tiles (bulk copy)
//   warp 1      : lane 0 issues the MMAs and the commits
//   warps 2..5  : gather the B rows (cp.async) and dequantise A into TMEM
//   warps 6..9  : epilogue (TMEM -> registers -> scales / SwiGLU -> bf16)
// Every wait is bounded: a role that waits ~1 s raises an abort flag, all
// roles drain what they issued, TMEM is freed and the error word is set.
#include "qmoe_internal.cuh"

namespace qmoe {
namespace {

constexpr int kThreads = 320;
constexpr int kRawSlot = 16384;
constexpr int kTabMax = kMaxE + kMaxShared + 1;
constexpr uint32_t kTmemCols = 512;

template <int BN>
struct Cfg {
  static constexpr int SA = BN >= 128 ? 4 : (BN >= 64 ? 6 : 7);   // A/B stages (TMEM + smem)
  static constexpr int R = BN >= 128 ? 3 : (BN >= 64 ? 6 : 8);    // raw weight ring
  static constexpr int B_STAGE = BN * 256;                        // BN rows x 128 K bf16
  static constexpr int STAGING = BN * 256;                        // epilogue staging
  static constexpr int A_COL0 = 2 * BN;                           // TMEM: acc0, acc1, then A stages
  static constexpr int OFF_B = 0;
  static constexpr int OFF_RAW = OFF_B + SA * B_STAGE;
  static constexpr int OFF_STG = OFF_RAW + R * kRawSlot;
  static constexpr int OFF_TAB = OFF_STG + STAGING;
  static constexpr int OFF_BAR = (OFF_TAB + 3 * kTabMax * 4 + 127) & ~127;  // mbarriers: 8-byte aligned
  static constexpr int NUM_BARS = 2 * SA + 2 * R + 4 + 1;
  static constexpr int OFF_MISC = (OFF_BAR + NUM_BARS * 8 + 15) & ~15;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;               // + alignment slack
  static_assert(OFF_BAR % 8 == 0 && OFF_MISC % 16 == 0, "barrier alignment");
  static_assert(OFF_RAW % 1024 == 0 && OFF_STG % 16 == 0 && B_STAGE % 1024 == 0, "buffer alignment");
  static_assert(A_COL0 + SA * 64 <= (int)kTmemCols, "TMEM budget");
  static_assert(SMEM <= 232448, "shared memory budget");
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

// ---- dequantisation to bf16 pairs ------------------------------------------
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

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + __expf(-g)); }

__device__ __forceinline__ uint16_t f2bf(float f) {
  const __nv_bfloat16 b = __float2bfloat16_rn(f);
  return *reinterpret_cast<const uint16_t*>(&b);
}

template <int BN, int MAT>
__global__ void __launch_bounds__(kThreads, 1) grouped_gemm_kernel(const GemmArgs a) {
  using C = Cfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sB = smem + C::OFF_B;
  uint8_t* sRaw = smem + C::OFF_RAW;
  uint8_t* sStg = smem + C::OFF_STG;
  int32_t* tab_off = reinterpret_cast<int32_t*>(smem + C::OFF_TAB);
  int32_t* s_seg_off = tab_off + kTabMax;
  int32_t* s_seg_cnt = s_seg_off + kTabMax;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* full = bars;                      // [SA] B gathered + A in TMEM
  uint64_t* empty = full + C::SA;             // [SA] MMA done with stage
  uint64_t* raw_full = empty + C::SA;         // [R] raw tile landed
  uint64_t* raw_empty = raw_full + C::R;      // [R] raw tile consumed
  uint64_t* acc_full = raw_empty + C::R;      // [2]
  uint64_t* acc_empty = acc_full + 2;         // [2]
  uint64_t* drain = acc_empty + 2;            // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_seg = a.n_seg;
  const int KS = a.K / kBK;

  for (int i = tid; i <= n_seg; i += kThreads) {
    tab_off[i] = a.tile_off[i];
    if (i < n_seg) {
      s_seg_off[i] = a.seg_off[i];
      s_seg_cnt[i] = a.seg_cnt[i];
    }
  }
  if (tid == 0) {
    for (int s = 0; s < C::SA; ++s) {
      mbar_init(&full[s], 256);
      mbar_init(&empty[s], 1);
    }
    for (int r = 0; r < C::R; ++r) {
      mbar_init(&raw_full[r], 1);
      mbar_init(&raw_empty[r], 128);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = tab_off[n_seg];

  if (warp == 0) {
    // ---------------- raw weight producer ----------------
    uint32_t rc = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
      const Tile t = decode_tile(tile, tab_off, s_seg_off, s_seg_cnt, n_seg, BN);
      const ExpertDev& ex = a.experts[t.seg];
      const int sb = stage_bytes(ex.fmt);
      const uint8_t* src = ex.w[MAT] + (size_t)t.mb * KS * sb;
      for (int ks = 0; ks < KS; ++ks) {
        const int slot = rc % C::R;
        ok = __all_sync(0xffffffffu, mbar_wait(&raw_empty[slot], ((rc / C::R) & 1) ^ 1, abort_flag));
        if (!ok) break;
        if (lane == 0) {
          mbar_arrive_expect_tx(&raw_full[slot], sb);
          bulk_g2s(sRaw + slot * kRawSlot, src + (size_t)ks * sb, sb, &raw_full[slot]);
        }
        ++rc;
        __syncwarp();
      }
    }
    // wait for copies that may still be in flight before the CTA can exit
    if (lane == 0) {
      const uint32_t first = rc > (uint32_t)C::R ? rc - C::R : 0;
      for (uint32_t i = first; i < rc; ++i) mbar_wait_drain(&raw_full[i % C::R], (i / C::R) & 1);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    uint32_t sc = 0, tc = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++tc) {
      const Tile t = decode_tile(tile, tab_off, s_seg_off, s_seg_cnt, n_seg, BN);
      const int b = tc & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&acc_empty[b], ((tc >> 1) & 1) ^ 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      const int n_mma = max(16, (t.nvalid + 15) & ~15);
      const uint32_t idesc = idesc_bf16_m128(n_mma);
      const uint32_t d_tmem = tmem_base + b * BN;
      for (int ks = 0; ks < KS; ++ks, ++sc) {
        const int s = sc % C::SA;
        ok = __all_sync(0xffffffffu, mbar_wait(&full[s], (sc / C::SA) & 1, abort_flag));
        if (!ok) break;
        tc_fence_after();
        if (lane == 0) {
          fence_proxy_async_smem();
          const uint32_t bbase = smem_u32(sB + s * C::B_STAGE);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t a_tmem = tmem_base + C::A_COL0 + s * 64 + kk * 8;
            const uint64_t bdesc = smem_desc_sw128(bbase + (kk >> 2) * (BN * 128) + (kk & 3) * 32);
            mma_bf16_ts(d_tmem, a_tmem, bdesc, idesc, (ks | kk) != 0);
          }
          mma_commit(&empty[s]);
        }
        __syncwarp();
      }
      if (!ok) break;
      if (lane == 0) mma_commit(&acc_full[b]);
      __syncwarp();
    }
    if (!ok) {
      // let every MMA issued so far finish before TMEM is released
      if (lane == 0) {
        mma_commit(drain);
        mbar_wait_drain(drain, 0);
      }
      __syncwarp();
    }
  } else if (warp < 6) {
    // ---------------- B gather + A dequantisation ----------------
    const int dq = tid - 64;                 // 0..127
    const int q = warp & 3;                  // TMEM lane quarter
    const int r = 32 * q + lane;             // weight row of the tile
    const int ch = dq & 15;                  // 16-byte chunk of a 256-byte B row
    const int katom = ch >> 3, cc = ch & 7;
    constexpr int RPT = BN / 8;              // B rows per thread
    uint32_t sc = 0, rc = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
      const Tile t = decode_tile(tile, tab_off, s_seg_off, s_seg_cnt, n_seg, BN);
      const int fmt = a.experts[t.seg].fmt;
      const uint16_t* srcp[RPT];
      uint32_t srcn[RPT];
#pragma unroll
      for (int i = 0; i < RPT; ++i) {
        const int n = (dq >> 4) + 8 * i;
        if (n < t.nvalid) {
          const int row = a.gather ? a.gather[t.row0 + n] : t.row0 + n;
          srcp[i] = a.act + (size_t)row * a.act_ld + ch * 8;
          srcn[i] = 16;
        } else {
          srcp[i] = a.act;
          srcn[i] = 0;
        }
      }
      for (int ks = 0; ks < KS; ++ks, ++sc, ++rc) {
        const int s = sc % C::SA;
        ok = __all_sync(0xffffffffu, mbar_wait(&empty[s], ((sc / C::SA) & 1) ^ 1, abort_flag));
        if (!ok) break;
        const uint32_t bst = smem_u32(sB + s * C::B_STAGE) + katom * (BN * 128);
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
          const int n = (dq >> 4) + 8 * i;
          cp_async16(bst + n * 128 + ((cc ^ (n & 7)) << 4), srcp[i] + (size_t)ks * kBK, srcn[i]);
        }
        cp_async_arrive_noinc(&full[s]);

        const int slot = rc % C::R;
        ok = __all_sync(0xffffffffu, mbar_wait(&raw_full[slot], (rc / C::R) & 1, abort_flag));
        if (!ok) break;
        const uint8_t* rawp = sRaw + slot * kRawSlot;
        uint32_t av[64];
        if (fmt == QMOE_W_INT4_G128) {
          uint4 wv[4];
#pragma unroll
          for (int c = 0; c < 4; ++c)
            wv[c] = *reinterpret_cast<const uint4*>(rawp + r * 64 + ((c ^ ((r >> 1) & 3)) << 4));
          const uint32_t sbits = reinterpret_cast<const uint16_t*>(rawp + 128 * 64)[r];
          mbar_arrive(&raw_empty[slot]);
          const uint32_t s2 = sbits | (sbits << 16);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            deq_int4_word(wv[c].x, s2, &av[16 * c + 0]);
            deq_int4_word(wv[c].y, s2, &av[16 * c + 4]);
            deq_int4_word(wv[c].z, s2, &av[16 * c + 8]);
            deq_int4_word(wv[c].w, s2, &av[16 * c + 12]);
          }
        } else {
          uint4 wv[8];
#pragma unroll
          for (int c = 0; c < 8; ++c)
            wv[c] = *reinterpret_cast<const uint4*>(rawp + r * 128 + ((c ^ (r & 7)) << 4));
          mbar_arrive(&raw_empty[slot]);
          if (fmt == QMOE_W_FP8_E4M3_PC) {
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              deq_fp8_word(wv[c].x, &av[8 * c + 0]);
              deq_fp8_word(wv[c].y, &av[8 * c + 2]);
              deq_fp8_word(wv[c].z, &av[8 * c + 4]);
              deq_fp8_word(wv[c].w, &av[8 * c + 6]);
            }
          } else {
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              deq_int8_word(wv[c].x, &av[8 * c + 0]);
              deq_int8_word(wv[c].y, &av[8 * c + 2]);
              deq_int8_word(wv[c].z, &av[8 * c + 4]);
              deq_int8_word(wv[c].w, &av[8 * c + 6]);
            }
          }
        }
        const uint32_t taddr = tmem_base + ((uint32_t)(32 * q) << 16) + C::A_COL0 + s * 64;
        tmem_st16(taddr + 0, &av[0]);
        tmem_st16(taddr + 16, &av[16]);
        tmem_st16(taddr + 32, &av[32]);
        tmem_st16(taddr + 48, &av[48]);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&full[s]);
      }
    }
    cp_async_wait_all();
  } else {
    // ---------------- epilogue ----------------
    // Each warp owns 32 accumulator rows (TMEM lane quarter q) and stages and
    // stores its own slice of the output rows, so only warp-level syncs are
    // needed.  mat 0: 16 intermediate columns (32 B) per token;
    // mat 1: 32 output columns (64 B) per token.
    const int q = warp & 3;
    const int r = 32 * q + lane;             // accumulator row = tile weight row
    constexpr int WCOLS = MAT == 0 ? 16 : 32;
    uint16_t* stg = reinterpret_cast<uint16_t*>(sStg) + (size_t)q * BN * WCOLS;
    uint32_t tc = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++tc) {
      const Tile t = decode_tile(tile, tab_off, s_seg_off, s_seg_cnt, n_seg, BN);
      const int b = tc & 1;
      const ExpertDev& ex = a.experts[t.seg];
      const float scale = ex.spc[MAT] ? ex.spc[MAT][t.mb * 128 + r] : 1.0f;
      ok = __all_sync(0xffffffffu, mbar_wait(&acc_full[b], (tc >> 1) & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      const int n_mma = max(16, (t.nvalid + 15) & ~15);
      const uint32_t taddr = tmem_base + ((uint32_t)(32 * q) << 16) + b * BN;
      for (int c0 = 0; c0 < n_mma; c0 += 16) {
        uint32_t v[16];
        tmem_ld16(taddr + c0, v);
        tmem_wait_ld();
        if (MAT == 0) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float f = __uint_as_float(v[i]) * scale;
            const float o = __shfl_xor_sync(0xffffffffu, f, 1);   // up value of the same index
            if ((lane & 1) == 0) stg[(c0 + i) * WCOLS + (lane >> 1)] = f2bf(silu_f(f) * o);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) stg[(c0 + i) * WCOLS + lane] = f2bf(__uint_as_float(v[i]) * scale);
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[b]);
      __syncwarp();
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

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
  if (tid == 0 && *abort_flag) atomicOr(a.err, kErrTimeout);
}

template <int BN>
cudaError_t launch_bn(const GemmArgs& a, int num_sms, cudaStream_t s) {
  using C = Cfg<BN>;
  auto kern = a.mat == 0 ? grouped_gemm_kernel<BN, 0> : grouped_gemm_kernel<BN, 1>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  kern<<<num_sms, kThreads, C::SMEM, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

bool gemm_bn_supported(int bn) { return bn == 16 || bn == 32 || bn == 64 || bn == 128; }

cudaError_t launch_grouped_gemm(const GemmArgs& a, int bn, int num_sms, cudaStream_t s) {
  switch (bn) {
    case 16: return launch_bn<16>(a, num_sms, s);
    case 32: return launch_bn<32>(a, num_sms, s);
    case 64: return launch_bn<64>(a, num_sms, s);
    case 128: return launch_bn<128>(a, num_sms, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace qmoe

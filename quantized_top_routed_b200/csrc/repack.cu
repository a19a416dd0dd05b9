// Weight re-layout at create time: the caller's canonical row-major codes
// become tiles of 128 weight rows x 128 K ("stages") that the grouped GEMM
// streams with bulk copies.  The stages of one 128-row block form one
// contiguous range of memory, the even K stages first and then the odd ones
// (the grouped GEMM's two stage classes), so each class's stages of a block
// are contiguous and several of them arrive with one bulk copy.
//
// Row order inside a tile:
//   gate/up matrix (mat 0): tile row 2j is gate row 64*mb + j, tile row
//     2j+1 is the matching up row I + 64*mb + j, so the SwiGLU epilogue
//     finds gate and up of one intermediate index in neighbouring lanes;
//   down matrix (mat 1): tile row r is weight row 128*mb + r.
// Chunk order: the tile is stored chunk-major, 16-byte chunk c of row r at
// byte c * 2048 + r * 16, so the 32 rows of a warp read one chunk as 512
// contiguous bytes (one coalesced 16-byte load per lane).
// Byte order inside a chunk (chosen for the in-register dequantisation):
//   INT8 / FP8 (16 K elements per chunk): each 32-bit word holds K elements
//     (k0, k2, k1, k3) in bytes 0..3, so bytes {0,2} and {1,3} expand to
//     bf16 pairs (k0,k1), (k2,k3); FP8 for the fp16 MMA mode keeps the
//     natural order (k0, k1, k2, k3), one hardware conversion per 16 bits.
//   INT4 (32 K elements per chunk): each 32-bit word holds 8 K elements as
//     biased nibbles (q + 8); nibble n < 4 is element 2n, nibble n >= 4 is
//     element 2(n-4)+1, so (w >> 4j) & 0x000F000F yields the pair (2j, 2j+1).
//     The 128 bf16 group scales of the tile (one per row) follow the 8192
//     code bytes.
// Per-channel scales (INT8 / FP8) are written in tile-row order.
#include "qmoe_internal.cuh"

namespace qmoe {
namespace {

__device__ __forceinline__ int src_row_of(int mat, int mb, int r, int I) {
  if (mat == 0) return (r & 1) ? (I + mb * 64 + (r >> 1)) : (mb * 64 + (r >> 1));
  return mb * 128 + r;
}

__global__ void repack_kernel(int fmt, int mat, const uint8_t* __restrict__ w, const void* __restrict__ scale,
                              int MB, int K, int I, uint8_t* __restrict__ dst, float* __restrict__ dst_spc) {
  const int rg = blockIdx.x * blockDim.x + threadIdx.x;  // global tile row
  const int ks = blockIdx.y;
  if (rg >= MB * 128) return;
  const int mb = rg >> 7, r = rg & 127;
  const int KS = K / kBK;
  const int src = src_row_of(mat, mb, r, I);
  uint8_t* tile = dst + ((size_t)mb * KS + stage_position(ks, KS)) * stage_bytes(fmt);
  if (fmt == QMOE_W_INT4_G128) {
    const uint8_t* s = w + (size_t)src * (K / 2) + ks * 64;
    auto q_at = [&](int kk) -> uint32_t {  // biased code q + 8 of element kk of this stage
      const uint8_t b = s[kk >> 1];
      const uint32_t nib = (kk & 1) ? (b >> 4) : (b & 0xF);
      return (nib ^ 0x8u) & 0xFu;  // two's complement -> q + 8
    };
    for (int c = 0; c < 4; ++c) {
      uint32_t words[4];
      for (int m = 0; m < 4; ++m) {
        const int base = 32 * c + 8 * m;
        uint32_t v = 0;
        for (int n = 0; n < 8; ++n) {
          const int kk = base + (n < 4 ? 2 * n : 2 * (n - 4) + 1);
          v |= q_at(kk) << (4 * n);
        }
        words[m] = v;
      }
      uint4* o = reinterpret_cast<uint4*>(tile + c * 2048 + r * 16);
      *o = make_uint4(words[0], words[1], words[2], words[3]);
    }
    const uint16_t* sc = static_cast<const uint16_t*>(scale);
    reinterpret_cast<uint16_t*>(tile + 128 * 64)[r] = sc[(size_t)src * (K / 128) + ks];
  } else {
    const uint8_t* s = w + (size_t)src * K + ks * 128;
    for (int c = 0; c < 8; ++c) {
      uint32_t words[4];
      for (int m = 0; m < 4; ++m) {
        const uint8_t* p = s + 16 * c + 4 * m;
        words[m] = fmt == kFmtFp8F16
                       ? ((uint32_t)p[0] | ((uint32_t)p[1] << 8) | ((uint32_t)p[2] << 16) | ((uint32_t)p[3] << 24))
                       : ((uint32_t)p[0] | ((uint32_t)p[2] << 8) | ((uint32_t)p[1] << 16) | ((uint32_t)p[3] << 24));
      }
      uint4* o = reinterpret_cast<uint4*>(tile + c * 2048 + r * 16);
      *o = make_uint4(words[0], words[1], words[2], words[3]);
    }
    if (ks == 0) dst_spc[rg] = static_cast<const float*>(scale)[src];
  }
}

}  // namespace

// rows: weight rows of the canonical matrix (2I for mat 0, d for mat 1).
cudaError_t launch_repack(int fmt, int mat, const void* w, const void* scale, int rows, int K, int I, uint8_t* dst,
                          float* dst_spc, cudaStream_t s) {
  const int MB = rows / 128;
  dim3 grid((MB * 128 + 127) / 128, K / kBK);
  repack_kernel<<<grid, 128, 0, s>>>(fmt, mat, static_cast<const uint8_t*>(w), scale, MB, K, I, dst, dst_spc);
  return cudaGetLastError();
}

}  // namespace qmoe

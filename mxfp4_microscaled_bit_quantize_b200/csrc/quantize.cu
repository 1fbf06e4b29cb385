// MXFP4 block quantizer kernels (bf16 -> packed E2M1 codes + E8M0 scales).
//
// Method: "Quantization Error" page, section "Where the error comes from" (one rounding step
// onto eight E2M1 magnitudes, an exact power-of-two scale per block, no dependence on block
// order) and the MXAttention abstract (Universal Optimal Scaling, Qmax = 7.25, next to the OCP
// rule). Each 32-element block: amax -> shared exponent (OCP or UOS) -> x * 2^-e rounded to
// nearest-even on the E2M1 grid, saturating at 6, by the hardware conversion
// cvt.rn.satfinite.e2m1x2.f32.
//
// Kernels:
//  * quantize_rows_kernel: blocks along the contiguous axis (Q, K, the standalone tensor). One
//    thread owns one whole block: four 16-byte loads, a thread-local amax, one 16-byte store of
//    codes. A warp therefore reads 2 KiB and writes 512 B of codes per step, fully coalesced.
//  * quantize_cols_kernel: blocks along the row axis of a [R, C] matrix, written transposed as
//    [C, R/2] codes (V along keys). Each thread loads two adjacent columns of 64 rows straight
//    from global memory (4-byte loads, 128 contiguous bytes per warp load), quantizes the four
//    32-row blocks and writes 32 contiguous bytes of codes per column.
//  * quantize_qkv_kernel: both of the above for one attention call (Q and K along d, V
//    transposed) in a single launch, so that the whole quantization pass is one kernel.
//
// Scale placement: row-major [.., rows, blocks] (the library's canonical layout), or the tile
// layout the block-scaled tensor-core MMA consumes: per 128-row tile and 4 blocks along K, a
// 512-byte atom where the byte of (row r, block k) sits at (r % 32) * 16 + (r / 32) * 4 + k.
#include <cuda_bf16.h>
#include <cstdint>

#include "mxattn_internal.h"
#include "sm100_ptx.cuh"

namespace mxattn {

__device__ __forceinline__ uint32_t atom_offset(uint32_t r128, uint32_t k4) {
  return (r128 & 31u) * 16u + (r128 >> 5) * 4u + k4;
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4& raw, float* v) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ uint32_t ld_stream_u32(const void* p) {
  uint32_t r;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(r) : "l"(p));
  return r;
}

__device__ __forceinline__ uint4 ld_stream_u4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Quantize 32 fp32 values (one block) into 16 code bytes and return the scale byte.
__device__ __forceinline__ uint32_t quantize_block32(float* v, int mode, uint4& codes) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const uint32_t byte = e8m0_scale_byte(amax, mode);
  const float inv = inv_pow2_from_byte(byte);
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] *= inv;   // exact: power of two
  codes.x = cvt_e2m1x8(v);
  codes.y = cvt_e2m1x8(v + 8);
  codes.z = cvt_e2m1x8(v + 16);
  codes.w = cvt_e2m1x8(v + 24);
  return byte;
}

// One 32-element block (global block index g over heads x rows_pad x kb) of the row quantizer.
__device__ __forceinline__ void quantize_rows_block(const RowQuantParams& p, uint32_t g) {
  const uint32_t row_bytes = p.kb * 16u;
  const uint32_t row = g / p.kb;               // head * rows_pad + n
  const uint32_t kbi = g - row * p.kb;
  const uint32_t head = row / p.rows_pad;
  const uint32_t n = row - head * p.rows_pad;
  float v[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = 0.f;
  if (n < p.rows) {
    const uint64_t src_row = static_cast<uint64_t>(head) * p.rows + n;
    const __nv_bfloat16* src = p.x + src_row * p.cols + static_cast<uint64_t>(kbi) * 32u;
    const uint32_t c0 = kbi * 32u;
    if (p.vec_ok && c0 + 32u <= p.cols) {
#pragma unroll
      for (int c = 0; c < 4; ++c) bf16x8_to_f32(ld_stream_u4(src + 8 * c), v + 8 * c);
    } else {
      for (uint32_t i = 0; i < 32u && c0 + i < p.cols; ++i) v[i] = __bfloat162float(src[i]);
    }
  }
  uint4 codes;
  const uint32_t byte = quantize_block32(v, p.mode, codes);
  *reinterpret_cast<uint4*>(p.codes + static_cast<uint64_t>(row) * row_bytes + kbi * 16u) = codes;
  uint64_t so;
  if (p.sf_layout == kSfRowMajor) {
    so = static_cast<uint64_t>(row) * p.kb + kbi;
  } else {
    const uint32_t tiles = p.rows_pad >> 7;
    const uint32_t katoms = (p.kb + 3u) >> 2;
    const uint64_t atom = (static_cast<uint64_t>(head) * tiles + (n >> 7)) * katoms + (kbi >> 2);
    so = atom * 512u + atom_offset(n & 127u, kbi & 3u);
  }
  p.scales[so] = static_cast<uint8_t>(byte);
}

__global__ void __launch_bounds__(256) quantize_rows_kernel(RowQuantParams p) {
  const uint32_t total = p.heads * p.rows_pad * p.kb;   // blocks
  for (uint32_t g = blockIdx.x * blockDim.x + threadIdx.x; g < total; g += gridDim.x * blockDim.x)
    quantize_rows_block(p, g);
}

// quantize_cols_kernel: each thread owns two adjacent columns (channels) and 64 rows (keys), i.e.
// two 32-row blocks per column. It issues 64 independent 4-byte loads (one bf16 pair per row; a
// warp's load covers 128 contiguous bytes of one row), then quantizes its four blocks and writes
// 32 contiguous bytes of codes per column (whole 32-byte sectors) and the two scale bytes of each
// column with one store. No shared memory and no CTA barrier: the loads of every warp are in
// flight together. A CTA of 8 warps covers 256 rows x 128 columns (2 column groups x 4 row
// groups); grid.y walks wider matrices in steps of 128 columns.
constexpr int kColRowsPerThread = 64;
constexpr int kColCtaRows = 256;
constexpr int kColCtaCols = 128;

// The work of one CTA (bx, by, bz) of the transposing quantizer.
__device__ __forceinline__ void quantize_cols_cta(const ColQuantParams& p, uint32_t bx, uint32_t by, uint32_t bz) {
  const uint32_t head = bz;
  const uint32_t warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t col = by * kColCtaCols + (warp & 1) * 64 + 2 * lane;   // this thread's first column
  const uint32_t r0 = bx * kColCtaRows + (warp >> 1) * kColRowsPerThread;
  const uint32_t blk0 = r0 >> 5;                      // absolute block index along rows
  if (col >= p.cols || blk0 >= p.nblk) return;
  const bool two = col + 1 < p.cols;
  const __nv_bfloat16* src = p.x + static_cast<uint64_t>(head) * p.rows * p.cols + col;
  // 4-byte loads need an even column count (then every (row, even column) pair is 4-byte aligned)
  const bool vec = p.vec_ok && (p.cols % 2u == 0u);
  uint32_t w[kColRowsPerThread];
#pragma unroll
  for (int i = 0; i < kColRowsPerThread; ++i) {
    const uint32_t r = r0 + i;
    w[i] = 0u;
    if (r < p.rows) {
      const __nv_bfloat16* e = src + static_cast<uint64_t>(r) * p.cols;
      if (vec) {
        w[i] = ld_stream_u32(e);
      } else {
        w[i] = __bfloat16_as_ushort(e[0]);
        if (two) w[i] |= static_cast<uint32_t>(__bfloat16_as_ushort(e[1])) << 16;
      }
    }
  }
  const bool second = blk0 + 1 < p.nblk;
#pragma unroll
  for (int cc = 0; cc < 2; ++cc) {
    if (cc == 1 && !two) break;
    uint4 codes[2];
    uint32_t bytes[2];
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      float v[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const uint32_t x = w[32 * b + i];
        v[i] = __uint_as_float(cc == 0 ? x << 16 : x & 0xFFFF0000u);
      }
      bytes[b] = quantize_block32(v, p.mode, codes[b]);
    }
    const uint32_t c = col + cc;
    uint8_t* dst = p.codes + (static_cast<uint64_t>(head) * p.cols + c) * (p.nblk * 16u) + blk0 * 16u;
    reinterpret_cast<uint4*>(dst)[0] = codes[0];
    if (second) reinterpret_cast<uint4*>(dst)[1] = codes[1];
    if (p.sf_layout == kSfRowMajor) {
      uint8_t* sc = p.scales + (static_cast<uint64_t>(head) * p.cols + c) * p.nblk + blk0;
      sc[0] = static_cast<uint8_t>(bytes[0]);
      if (second) sc[1] = static_cast<uint8_t>(bytes[1]);
    } else {
      // atom per (head, 128-row tile, 128-column group); MN index = column, K index = block; the
      // two blocks are K indices blk0 & 3 and (blk0 & 3) + 1, adjacent bytes (blk0 is even)
      const uint32_t tiles = p.nblk >> 2;             // nblk is a multiple of 4 here
      const uint32_t cgroups = (p.cols + 127u) >> 7;
      const uint64_t atom = (static_cast<uint64_t>(head) * tiles + (blk0 >> 2)) * cgroups + (c >> 7);
      uint8_t* sc = p.scales + atom * 512u + atom_offset(c & 127u, blk0 & 3u);
      *reinterpret_cast<uint16_t*>(sc) = static_cast<uint16_t>(bytes[0] | ((second ? bytes[1] : 0u) << 8));
    }
  }
}

__global__ void __launch_bounds__(256) quantize_cols_kernel(ColQuantParams p) {
  quantize_cols_cta(p, blockIdx.x, blockIdx.y, blockIdx.z);
}

// Q and K along d and V transposed in one launch: CTAs [0, v_ctas) are the transposing
// quantizer's grid (flattened), the rest walk the Q blocks and then the K blocks grid-stride.
__global__ void __launch_bounds__(256) quantize_qkv_kernel(QkvQuantParams p) {
  if (blockIdx.x < p.v_ctas) {
    const uint32_t bx = blockIdx.x % p.v_gx, rest = blockIdx.x / p.v_gx;
    quantize_cols_cta(p.v, bx, rest % p.v_gy, rest / p.v_gy);
    return;
  }
  const uint32_t nq = p.q.heads * p.q.rows_pad * p.q.kb, nk = p.k.heads * p.k.rows_pad * p.k.kb;
  const uint32_t stride = (gridDim.x - p.v_ctas) * blockDim.x;
  for (uint32_t g = (blockIdx.x - p.v_ctas) * blockDim.x + threadIdx.x; g < nq + nk; g += stride) {
    if (g < nq) quantize_rows_block(p.q, g);
    else quantize_rows_block(p.k, g - nq);
  }
}

// NVFP4 (comparison format): blocks of 16 along the contiguous axis, scale s = E4M3(amax / 6),
// elements x / s on the E2M1 grid; both quotients are correctly rounded fp32 divisions, so the
// grid decisions are taken on the same fp32 values the oracle takes them on. One thread per block.
// amax -> E4M3 scale byte -> codes of x / s (zero block when the scale rounds to 0)
__device__ __forceinline__ uint32_t nvfp4_block16(float* v, uint2& codes) {
  float amax = 0.f;
#pragma unroll
  for (int k = 0; k < 16; ++k) amax = fmaxf(amax, fabsf(v[k]));
  const uint32_t byte = e4m3_byte(__fdiv_rn(amax, 6.0f));
  const float s = e4m3_value(byte);
#pragma unroll
  for (int k = 0; k < 16; ++k) v[k] = (s > 0.f) ? __fdiv_rn(v[k], s) : 0.f;
  codes = make_uint2(cvt_e2m1x8(v), cvt_e2m1x8(v + 8));
  return byte;
}

__global__ void __launch_bounds__(256) quantize_rows_nvfp4_kernel(const NvQuantParams p) {
  const uint32_t nb = (p.cols + 15u) / 16u;
  const uint32_t rows_pad = p.rows_pad > p.rows ? p.rows_pad : p.rows;
  const uint64_t total = static_cast<uint64_t>(p.heads) * rows_pad * nb;
  const uint64_t stride = static_cast<uint64_t>(gridDim.x) * blockDim.x;
  for (uint64_t i = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
    const uint64_t prow = i / nb;                       // padded row index over all heads
    const uint32_t blk = static_cast<uint32_t>(i - prow * nb);
    const uint64_t head = prow / rows_pad;
    const uint32_t n = static_cast<uint32_t>(prow - head * rows_pad);
    const uint32_t c0 = blk * 16u;
    uint2 codes = make_uint2(0u, 0u);
    uint32_t byte = 0;
    if (n < p.rows) {
      const __nv_bfloat16* src = p.x + (head * p.rows + n) * p.cols + c0;
      float v[16];
      if (p.vec_ok && c0 + 16u <= p.cols) {
        const uint4 r0 = ld_stream_u4(src), r1 = ld_stream_u4(src + 8);
        bf16x8_to_f32(r0, v);
        bf16x8_to_f32(r1, v + 8);
      } else {
#pragma unroll
        for (int k = 0; k < 16; ++k) v[k] = (c0 + k < p.cols) ? __bfloat162float(src[k]) : 0.f;
      }
      byte = nvfp4_block16(v, codes);
    }
    *reinterpret_cast<uint2*>(p.codes + prow * (nb * 8u) + blk * 8u) = codes;
    if (p.sf_layout == kSfRowMajor) {
      p.scales[prow * nb + blk] = static_cast<uint8_t>(byte);
    } else {
      const uint32_t ksteps = (nb + 3u) / 4u;
      const uint64_t atom = (head * (rows_pad / 128u) + (n >> 7)) * ksteps + (blk >> 2);
      p.scales[atom * 512u + atom_offset(n & 127u, blk & 3u)] = static_cast<uint8_t>(byte);
    }
  }
}

// One thread per (head, 16-row block, column), columns fastest: the warp's strided loads of one
// row segment are contiguous across lanes.
__global__ void __launch_bounds__(256) quantize_cols_nvfp4_kernel(const NvColQuantParams p) {
  const uint32_t nblk = p.rows_pad / 16u;
  const uint64_t total = static_cast<uint64_t>(p.heads) * nblk * p.cols;
  const uint64_t stride = static_cast<uint64_t>(gridDim.x) * blockDim.x;
  for (uint64_t i = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
    const uint32_t col = static_cast<uint32_t>(i % p.cols);
    const uint64_t hb = i / p.cols;
    const uint32_t blk = static_cast<uint32_t>(hb % nblk);
    const uint64_t head = hb / nblk;
    const uint32_t r0 = blk * 16u;
    uint2 codes = make_uint2(0u, 0u);
    uint32_t byte = 0;
    if (r0 < p.rows) {
      float v[16];
      const __nv_bfloat16* src = p.x + (head * p.rows + r0) * p.cols + col;
#pragma unroll
      for (int k = 0; k < 16; ++k) v[k] = (r0 + k < p.rows) ? __bfloat162float(src[static_cast<size_t>(k) * p.cols]) : 0.f;
      byte = nvfp4_block16(v, codes);
    }
    *reinterpret_cast<uint2*>(p.codes + (head * p.cols + col) * (nblk * 8u) + blk * 8u) = codes;
    const uint64_t atom = head * (p.rows_pad / 64u) + (blk >> 2);
    p.scales[atom * 512u + atom_offset(col & 127u, blk & 3u)] = static_cast<uint8_t>(byte);
  }
}

cudaError_t launch_quantize_cols_nvfp4(const NvColQuantParams& p, cudaStream_t stream) {
  const uint64_t total = static_cast<uint64_t>(p.heads) * (p.rows_pad / 16u) * p.cols;
  if (total == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const uint64_t want = (total + 255) / 256;
  const uint64_t cap = static_cast<uint64_t>(sms) * 16;
  quantize_cols_nvfp4_kernel<<<static_cast<unsigned>(want < cap ? want : cap), 256, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_quantize_rows_nvfp4(const NvQuantParams& p, cudaStream_t stream) {
  const uint32_t rows_pad = p.rows_pad > p.rows ? p.rows_pad : p.rows;
  const uint64_t total = static_cast<uint64_t>(p.heads) * rows_pad * ((p.cols + 15u) / 16u);
  if (total == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const uint64_t want = (total + 255) / 256;
  const uint64_t cap = static_cast<uint64_t>(sms) * 8;
  quantize_rows_nvfp4_kernel<<<static_cast<unsigned>(want < cap ? want : cap), 256, 0, stream>>>(p);
  return cudaGetLastError();
}

// One thread per atom byte: invert atom_offset to find the (row, block) it holds.
__global__ void __launch_bounds__(256) repack_scales_kernel(const ScaleRepackParams p) {
  const uint32_t kgroups = p.kgroups ? p.kgroups : 1u;
  const uint64_t total = static_cast<uint64_t>(p.heads) * p.tiles * kgroups * 512u;
  const uint64_t stride = static_cast<uint64_t>(gridDim.x) * blockDim.x;
  for (uint64_t i = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
    const uint32_t b = static_cast<uint32_t>(i & 511u);
    const uint64_t atom = i >> 9;
    const uint32_t g = static_cast<uint32_t>(atom % kgroups);
    const uint32_t t = static_cast<uint32_t>((atom / kgroups) % p.tiles);
    const uint64_t head = atom / kgroups / p.tiles;
    const uint32_t r = ((b >> 4) & 31u) + 32u * ((b & 15u) >> 2);   // 0..127
    const uint32_t k = b & 3u;
    uint8_t v = 0;
    if (!p.transposed) {
      const uint32_t row = t * 128u + r;
      const uint32_t blk = g * 4u + k;
      if (row < p.rows && blk < p.kb) v = p.src[(head * p.rows + row) * p.kb + blk];
    } else {
      const uint32_t blk = t * 4u + k;
      if (r < p.rows && blk < p.kb) v = p.src[(head * p.rows + r) * p.kb + blk];
    }
    p.dst[i] = v;
  }
}

cudaError_t launch_repack_scales(const ScaleRepackParams& p, cudaStream_t stream) {
  const uint64_t total = static_cast<uint64_t>(p.heads) * p.tiles * (p.kgroups ? p.kgroups : 1u) * 512u;
  if (total == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const uint64_t want = (total + 255) / 256;
  const uint64_t cap = static_cast<uint64_t>(sms) * 8;
  repack_scales_kernel<<<static_cast<unsigned>(want < cap ? want : cap), 256, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_quantize_rows(const RowQuantParams& p, cudaStream_t stream) {
  const uint64_t total = static_cast<uint64_t>(p.heads) * p.rows_pad * p.kb;
  if (total == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const uint64_t want = (total + 255) / 256;
  const uint64_t cap = static_cast<uint64_t>(sms) * 8;
  const unsigned grid = static_cast<unsigned>(want < cap ? want : cap);
  quantize_rows_kernel<<<grid, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_quantize_qkv(const RowQuantParams& q, const RowQuantParams& k, const ColQuantParams& v,
                               cudaStream_t stream) {
  QkvQuantParams p{q, k, v, 0, 0, 0};
  p.v_gx = (v.nblk * 32u + kColCtaRows - 1) / kColCtaRows;
  p.v_gy = (v.cols + kColCtaCols - 1) / kColCtaCols;
  const uint64_t v_ctas = (v.heads == 0 || v.cols == 0 || v.nblk == 0)
                              ? 0 : static_cast<uint64_t>(p.v_gx) * p.v_gy * v.heads;
  const uint64_t row_blocks = static_cast<uint64_t>(q.heads) * q.rows_pad * q.kb +
                              static_cast<uint64_t>(k.heads) * k.rows_pad * k.kb;
  if (v_ctas + row_blocks == 0) return cudaSuccess;
  if (v_ctas >= (1ull << 31) || row_blocks >= (1ull << 32)) return cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const uint64_t want = (row_blocks + 255) / 256;
  const uint64_t cap = static_cast<uint64_t>(sms) * 8;
  const uint64_t row_ctas = want < cap ? want : cap;
  p.v_ctas = static_cast<uint32_t>(v_ctas);
  quantize_qkv_kernel<<<static_cast<unsigned>(v_ctas + row_ctas), 256, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_quantize_cols(const ColQuantParams& p, cudaStream_t stream) {
  if (p.heads == 0 || p.cols == 0 || p.nblk == 0) return cudaSuccess;
  dim3 grid((p.nblk * 32u + kColCtaRows - 1) / kColCtaRows, (p.cols + kColCtaCols - 1) / kColCtaCols, p.heads);
  quantize_cols_kernel<<<grid, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace mxattn

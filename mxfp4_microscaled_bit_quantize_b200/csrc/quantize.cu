// MXFP4 block quantizer kernels (bf16 -> packed E2M1 codes + E8M0 scales).
//
// Method: "Quantization Error" page, section "Where the error comes from" (one rounding step
// onto eight E2M1 magnitudes, an exact power-of-two scale per block, no dependence on block
// order) and the MXAttention abstract (Universal Optimal Scaling, Qmax = 7.25, next to the OCP
// rule). Each 32-element block: amax -> shared exponent (OCP or UOS) -> x * 2^-e rounded to
// nearest-even on the E2M1 grid, saturating at 6, by the hardware conversion
// cvt.rn.satfinite.e2m1x2.f32.
//
// Two kernels:
//  * quantize_rows_kernel: blocks along the contiguous axis (Q, K, the standalone tensor). One
//    thread owns one whole block: four 16-byte loads, a thread-local amax, one 16-byte store of
//    codes. A warp therefore reads 2 KiB and writes 512 B of codes per step, fully coalesced.
//  * quantize_cols_kernel: blocks along the row axis of a [R, C] matrix, written transposed as
//    [C, R/2] codes (V along keys). A CTA stages 256 rows x 64 columns in shared memory; each
//    thread then quantizes two consecutive 32-row blocks of one column and writes 32 contiguous
//    bytes of codes.
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

__global__ void __launch_bounds__(256) quantize_rows_kernel(RowQuantParams p) {
  const uint32_t total = p.heads * p.rows_pad * p.kb;   // blocks
  const uint32_t row_bytes = p.kb * 16u;
  for (uint32_t g = blockIdx.x * blockDim.x + threadIdx.x; g < total; g += gridDim.x * blockDim.x) {
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
}

// Stage: 256 rows x 64 columns of bf16, row pitch 72 elements (144 B) so that the column reads
// of the compute phase (32 lanes on consecutive columns) hit distinct banks.
constexpr int kColTileRows = 256;
constexpr int kColTileCols = 64;
constexpr int kColPitch = 72;

__global__ void __launch_bounds__(256) quantize_cols_kernel(ColQuantParams p) {
  __shared__ __align__(16) __nv_bfloat16 tile[kColTileRows * kColPitch];
  const uint32_t head = blockIdx.z;
  const uint32_t r0 = blockIdx.x * kColTileRows;      // first row (key) of this tile
  const uint32_t c0 = blockIdx.y * kColTileCols;      // first column (channel)
  const __nv_bfloat16* src = p.x + static_cast<uint64_t>(head) * p.rows * p.cols;
  const int tid = threadIdx.x;

  // Load: each pass covers 32 rows x 64 columns, one 16-byte vector per thread.
#pragma unroll 4
  for (int pass = 0; pass < kColTileRows / 32; ++pass) {
    const uint32_t rr = pass * 32 + (tid >> 3);
    const uint32_t cc = (tid & 7) * 8;
    const uint32_t r = r0 + rr, c = c0 + cc;
    uint4 raw = make_uint4(0, 0, 0, 0);
    if (r < p.rows) {
      const __nv_bfloat16* s = src + static_cast<uint64_t>(r) * p.cols + c;
      if (p.vec_ok && c + 8 <= p.cols) {
        raw = ld_stream_u4(s);
      } else {
        uint16_t h[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        for (uint32_t i = 0; i < 8 && c + i < p.cols; ++i) h[i] = __bfloat16_as_ushort(s[i]);
        raw.x = h[0] | (uint32_t(h[1]) << 16);
        raw.y = h[2] | (uint32_t(h[3]) << 16);
        raw.z = h[4] | (uint32_t(h[5]) << 16);
        raw.w = h[6] | (uint32_t(h[7]) << 16);
      }
    }
    *reinterpret_cast<uint4*>(&tile[rr * kColPitch + cc]) = raw;
  }
  __syncthreads();

  // Compute: thread (column cl, pair kp) quantizes row blocks 2kp and 2kp+1 of its column.
  const uint32_t cl = tid & 63;
  const uint32_t kp = tid >> 6;
  const uint32_t col = c0 + cl;
  const uint32_t blk0 = (r0 >> 5) + 2 * kp;          // absolute block index along rows
  if (col >= p.cols || blk0 >= p.nblk) return;
  uint4 codes[2];
  uint32_t bytes[2];
#pragma unroll
  for (int b = 0; b < 2; ++b) {
    float v[32];
    const uint32_t rb = (2 * kp + b) * 32;
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __bfloat162float(tile[(rb + i) * kColPitch + cl]);
    bytes[b] = quantize_block32(v, p.mode, codes[b]);
  }
  const bool second = blk0 + 1 < p.nblk;
  uint8_t* dst = p.codes + (static_cast<uint64_t>(head) * p.cols + col) * (p.nblk * 16u) + blk0 * 16u;
  reinterpret_cast<uint4*>(dst)[0] = codes[0];
  if (second) reinterpret_cast<uint4*>(dst)[1] = codes[1];
  if (p.sf_layout == kSfRowMajor) {
    uint8_t* s = p.scales + (static_cast<uint64_t>(head) * p.cols + col) * p.nblk + blk0;
    s[0] = static_cast<uint8_t>(bytes[0]);
    if (second) s[1] = static_cast<uint8_t>(bytes[1]);
  } else {
    // atom per (head, 128-row tile, 128-column group); MN index = column, K index = block
    const uint32_t tiles = p.nblk >> 2;               // nblk is a multiple of 4 here
    const uint32_t cgroups = (p.cols + 127u) >> 7;
    const uint64_t atom = (static_cast<uint64_t>(head) * tiles + (blk0 >> 2)) * cgroups + (col >> 7);
    uint8_t* s = p.scales + atom * 512u + atom_offset(col & 127u, blk0 & 3u);
    s[0] = static_cast<uint8_t>(bytes[0]);
    if (second) s[1] = static_cast<uint8_t>(bytes[1]);
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

cudaError_t launch_quantize_cols(const ColQuantParams& p, cudaStream_t stream) {
  if (p.heads == 0 || p.cols == 0 || p.nblk == 0) return cudaSuccess;
  dim3 grid((p.nblk * 32u + kColTileRows - 1) / kColTileRows, (p.cols + kColTileCols - 1) / kColTileCols,
            p.heads);
  quantize_cols_kernel<<<grid, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace mxattn

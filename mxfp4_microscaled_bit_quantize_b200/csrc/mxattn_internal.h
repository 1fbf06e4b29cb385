// Internal declarations shared by the library's translation units (not part of the C ABI).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace mxattn {

// Keys per KV tile of the attention kernel: P~ is quantized with the running max in force at
// each tile, so this width is part of what the kernel computes (MXATTN_KV_TILE in mxattn.h).
constexpr int kKvTile = 128;

enum SfLayout : int { kSfRowMajor = 0, kSfAtom = 1 };

// Scale modes (MXATTN_SCALE_* in mxattn.h): MXFP4 with the OCP or the UOS exponent rule, or the
// NVFP4 comparison format.
enum : int { kModeOcp = 0, kModeUos = 1, kModeNvfp4 = 2 };

// Blocks of 32 along the contiguous axis of `heads` matrices of [rows, cols] bf16. Rows in
// [rows, rows_pad) are written as all-zero blocks (codes 0, scale byte 0).
struct RowQuantParams {
  const __nv_bfloat16* x;
  uint32_t heads, rows, rows_pad, cols, kb;   // kb = ceil(cols / 32)
  uint8_t* codes;                              // [heads][rows_pad][kb * 16]
  uint8_t* scales;                             // row-major [heads][rows_pad][kb] or atom tiles
  int mode;                                    // 0 = OCP, 1 = UOS
  int sf_layout;
  int vec_ok;                                  // cols % 8 == 0 and x 16-byte aligned
};

// Blocks of 32 along the row axis of `heads` matrices of [rows, cols] bf16, written
// transposed: codes [heads][cols][nblk * 16], nblk >= ceil(rows / 32) (extra blocks are zero).
struct ColQuantParams {
  const __nv_bfloat16* x;
  uint32_t heads, rows, cols, nblk;
  uint8_t* codes;
  uint8_t* scales;                             // row-major [heads][cols][nblk] or atom tiles
  int mode;
  int sf_layout;
  int vec_ok;
};

cudaError_t launch_quantize_rows(const RowQuantParams& p, cudaStream_t stream);
cudaError_t launch_quantize_cols(const ColQuantParams& p, cudaStream_t stream);

// Q and K (row quantizer) and V (transposing quantizer) of one attention call in a single launch.
struct QkvQuantParams {
  RowQuantParams q, k;
  ColQuantParams v;
  uint32_t v_ctas, v_gx, v_gy;    // the transposing quantizer's CTAs come first, grid (v_gx, v_gy, heads)
};
cudaError_t launch_quantize_qkv(const RowQuantParams& q, const RowQuantParams& k, const ColQuantParams& v,
                               cudaStream_t stream);

// NVFP4 (blocks of 16, E4M3 scales) along the contiguous axis: codes [heads*rows][ceil(cols/16)*8],
// scales [heads*rows][ceil(cols/16)].
// With sf_layout = kSfAtom: rows [rows, rows_pad) are zero (codes 0, scale 0) and the scales go to
// atoms [heads][rows_pad/128][ceil(cols/64)][512] (an atom: 128 rows x 4 blocks of 16).
struct NvQuantParams {
  const __nv_bfloat16* x;
  uint32_t heads, rows, cols;
  uint8_t* codes;
  uint8_t* scales;
  int vec_ok;                                  // cols % 8 == 0 and x 16-byte aligned
  uint32_t rows_pad;                           // >= rows (codes are [heads][rows_pad][nb * 8])
  int sf_layout;
};
cudaError_t launch_quantize_rows_nvfp4(const NvQuantParams& p, cudaStream_t stream);

// NVFP4 along the row axis of `heads` matrices [rows, cols] (V along keys), written transposed:
// codes [heads][cols][nblk * 8] with nblk = rows_pad / 16 blocks of 16 rows (blocks past `rows` are
// zero), scales as atoms [heads][rows_pad / 64][512] (MN index = column < 128, K index = block % 4).
struct NvColQuantParams {
  const __nv_bfloat16* x;
  uint32_t heads, rows, cols, rows_pad;
  uint8_t* codes;
  uint8_t* scales;
};
cudaError_t launch_quantize_cols_nvfp4(const NvColQuantParams& p, cudaStream_t stream);

// Row-major scale bytes -> 512-byte MMA atoms [heads][tiles][512], zero where the source has no
// element. transposed = 0: src [heads][rows][kb], atom t holds rows 128t.. and blocks 0..3;
// transposed = 1 (V^T): src [heads][rows = channels][kb = key blocks], atom t holds channels
// 0..127 and key blocks 4t..4t+3.
// kgroups > 1 (transposed = 0 only): atoms [heads][tiles][kgroups][512], kgroup g holding blocks
// 4g..4g+3 of the rows of its tile.
struct ScaleRepackParams {
  const uint8_t* src;
  uint8_t* dst;
  uint32_t heads, tiles, rows, kb;
  int transposed;
  uint32_t kgroups;
};
cudaError_t launch_repack_scales(const ScaleRepackParams& p, cudaStream_t stream);

struct AttnParams {
  const uint8_t* qsf;      // atom-tiled scales of Q  [B*Hq][Npad/128][512]
  const uint8_t* ksf;      // atom-tiled scales of K  [B*Hkv][Npad/128][512]
  const uint8_t* vsf;      // atom-tiled scales of V^T [B*Hkv][Npad/128][512]
  void* out;               // [B, Hq, N, d], fp32 or bf16
  int out_bf16;
  int B, Hq, Hkv, N, Npad, causal, mode, pnq;
  int rows_per_head;       // row stride between heads in the Q / K code tensors (Npad or N)
  float scale_log2;        // log2(e) / sqrt(d)
  unsigned int* status;    // device status word (0 = ok)
  uint8_t* dbg_codes;      // optional P~ dump: [r1 - r0][Npad / 2]
  uint8_t* dbg_scales;     //                  [r1 - r0][Npad / 32]
  int dbg_bh, dbg_r0, dbg_r1;
};

cudaError_t launch_attention(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                             const AttnParams& p, int d, cudaStream_t stream);

// Block-scaled MXFP4 GEMM C[M, N] = dq(A) dq(B)^T; A, B codes are read through tensor maps, their
// scales from atoms [row tile][kgroup][512] (kgroup = 128 K elements; B row tiles padded to even).
struct GemmParams {
  const uint8_t* sfa;
  const uint8_t* sfb;
  void* c;                 // [M, N] fp32 or bf16, row-major
  int M, N, K;
  int k_stages;            // ceil(K / 256)
  int kgroups;             // atoms per row tile (zero-padded past K): 2 * k_stages, NVFP4 4 * k_stages
  int out_bf16;
  int nvfp4;               // 0: MXFP4 (blocks of 32, UE8M0); 1: NVFP4 (blocks of 16, UE4M3)
  unsigned int* status;
};

cudaError_t launch_gemm(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmC, const GemmParams& p,
                        cudaStream_t stream);

// Status codes written by kernels into the workspace status word.
enum : unsigned int {
  kStatusTimeoutQ = 0x100,
  kStatusTimeoutKV = 0x200,
  kStatusTimeoutS = 0x300,
  kStatusTimeoutP = 0x400,
  kStatusTimeoutPV = 0x500,
  kStatusTimeoutEmpty = 0x600,
  kStatusSelfTest = 0x700,
};

cudaError_t launch_wait_timeout_selftest(unsigned int* status, unsigned int* seen, cudaStream_t stream);

}  // namespace mxattn

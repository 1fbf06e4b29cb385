// Host side of the C ABI declared in include/mxattn.h: argument checks, workspace carving,
// TMA tensor-map encoding and kernel launches. No device memory is allocated here.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/mxattn.h"
#include "mxattn_internal.h"

using namespace mxattn;

namespace {

constexpr size_t kAlign = 1024;
constexpr int kTile = 128;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct WsLayout {
  size_t qc, qs, kc, ks, vc, vs, total;
  int npad;
};

// status word at offset 0; every region 1 KiB aligned (TMA needs 16 B, bulk copies 16 B).
bool ws_layout(int B, int Hq, int Hkv, int N, int d, WsLayout* L) {
  if (B < 1 || Hq < 1 || Hkv < 1 || N < 1 || (d != 64 && d != 128) || Hq % Hkv != 0) return false;
  const size_t npad = align_up(static_cast<size_t>(N), kTile);
  const size_t tiles = npad / kTile;
  if (static_cast<uint64_t>(B) * Hq * tiles >= (1ull << 31)) return false;
  if (static_cast<uint64_t>(B) * Hq * npad >= (1ull << 31)) return false;
  size_t off = kAlign;  // status area
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, kAlign);
    return o;
  };
  L->qc = take(static_cast<size_t>(B) * Hq * npad * (d / 2));
  // scale regions sized for the larger format: NVFP4 has d / 64 atoms per 128 Q / K rows and one
  // V atom per 64 keys (MXFP4 uses the first 512 bytes per 128 rows or keys, packed)
  const size_t qk_atoms = (d >= 128) ? static_cast<size_t>(d / 64) : 1;
  L->qs = take(static_cast<size_t>(B) * Hq * tiles * qk_atoms * 512);
  L->kc = take(static_cast<size_t>(B) * Hkv * npad * (d / 2));
  L->ks = take(static_cast<size_t>(B) * Hkv * tiles * qk_atoms * 512);
  L->vc = take(static_cast<size_t>(B) * Hkv * d * (npad / 2));
  L->vs = take(static_cast<size_t>(B) * Hkv * tiles * 1024);
  L->total = off;
  L->npad = static_cast<int>(npad);
  return true;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }();
  return fn;
}

// 2-D uint8 tensor map over a row-major [rows, row_bytes] byte matrix, box [box_rows, box_bytes].
bool make_map(CUtensorMap* m, const void* base, uint64_t row_bytes, uint64_t rows, uint32_t box_bytes,
              uint32_t box_rows, CUtensorMapSwizzle swz) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {row_bytes, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_bytes, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2-D tensor map of the given element type over a row-major matrix (dims and box in elements).
bool make_map_typed(CUtensorMap* m, CUtensorMapDataType dtype, const void* base, uint64_t cols, uint64_t rows,
                    uint64_t row_bytes, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, dtype, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

mxattn_status prepare_impl(const void* q, const void* k, const void* v, int B, int Hq, int Hkv, int N, int d,
                           int scale_mode, void* ws, size_t ws_bytes, cudaStream_t st, const WsLayout& L) {
  uint8_t* w = static_cast<uint8_t*>(ws);
  if (d < kTile) {
    // scale atoms have room for 128 rows / 4 blocks; d = 64 leaves part of them unused
    if (cudaMemsetAsync(w + L.qs, 0, L.kc - L.qs, st) != cudaSuccess) return MXATTN_ERR_CUDA;
    if (cudaMemsetAsync(w + L.ks, 0, L.vc - L.ks, st) != cudaSuccess) return MXATTN_ERR_CUDA;
    if (cudaMemsetAsync(w + L.vs, 0, L.total - L.vs, st) != cudaSuccess) return MXATTN_ERR_CUDA;
  }
  if (scale_mode == kModeNvfp4) {
    NvQuantParams nq{};
    nq.x = static_cast<const __nv_bfloat16*>(q);
    nq.heads = static_cast<uint32_t>(B * Hq);
    nq.rows = static_cast<uint32_t>(N);
    nq.rows_pad = static_cast<uint32_t>(L.npad);
    nq.cols = static_cast<uint32_t>(d);
    nq.codes = w + L.qc;
    nq.scales = w + L.qs;
    nq.vec_ok = aligned(q, 16) ? 1 : 0;
    nq.sf_layout = kSfAtom;
    if (launch_quantize_rows_nvfp4(nq, st) != cudaSuccess) return MXATTN_ERR_CUDA;
    nq.x = static_cast<const __nv_bfloat16*>(k);
    nq.heads = static_cast<uint32_t>(B * Hkv);
    nq.codes = w + L.kc;
    nq.scales = w + L.ks;
    nq.vec_ok = aligned(k, 16) ? 1 : 0;
    if (launch_quantize_rows_nvfp4(nq, st) != cudaSuccess) return MXATTN_ERR_CUDA;
    NvColQuantParams vq{};
    vq.x = static_cast<const __nv_bfloat16*>(v);
    vq.heads = static_cast<uint32_t>(B * Hkv);
    vq.rows = static_cast<uint32_t>(N);
    vq.cols = static_cast<uint32_t>(d);
    vq.rows_pad = static_cast<uint32_t>(L.npad);
    vq.codes = w + L.vc;
    vq.scales = w + L.vs;
    if (launch_quantize_cols_nvfp4(vq, st) != cudaSuccess) return MXATTN_ERR_CUDA;
    return MXATTN_OK;
  }
  RowQuantParams rq{}, rk{};
  rq.x = static_cast<const __nv_bfloat16*>(q);
  rq.heads = static_cast<uint32_t>(B * Hq);
  rq.rows = static_cast<uint32_t>(N);
  rq.rows_pad = static_cast<uint32_t>(L.npad);
  rq.cols = static_cast<uint32_t>(d);
  rq.kb = static_cast<uint32_t>(d / 32);
  rq.codes = w + L.qc;
  rq.scales = w + L.qs;
  rq.mode = scale_mode;
  rq.sf_layout = kSfAtom;
  rq.vec_ok = aligned(q, 16) ? 1 : 0;
  rk = rq;
  rk.x = static_cast<const __nv_bfloat16*>(k);
  rk.heads = static_cast<uint32_t>(B * Hkv);
  rk.codes = w + L.kc;
  rk.scales = w + L.ks;
  rk.vec_ok = aligned(k, 16) ? 1 : 0;
  ColQuantParams cq{};
  cq.x = static_cast<const __nv_bfloat16*>(v);
  cq.heads = static_cast<uint32_t>(B * Hkv);
  cq.rows = static_cast<uint32_t>(N);
  cq.cols = static_cast<uint32_t>(d);
  cq.nblk = static_cast<uint32_t>(L.npad / 32);
  cq.codes = w + L.vc;
  cq.scales = w + L.vs;
  cq.mode = scale_mode;
  cq.sf_layout = kSfAtom;
  cq.vec_ok = aligned(v, 16) ? 1 : 0;
  // one launch for all three operands
  if (launch_quantize_qkv(rq, rk, cq, st) != cudaSuccess) return MXATTN_ERR_CUDA;
  (void)ws_bytes;
  return MXATTN_OK;
}

// Where the attention kernel reads its FP4 codes: the workspace (rows padded to Npad, V^T rows of
// Npad/2 bytes) or caller tensors in the canonical layout (N rows per head, V^T rows of
// ceil(N/32)*16 bytes). Rows and keys past N are never used: padded query rows are not stored,
// keys >= N are masked, and the tensor maps zero-fill reads past the last row or column.
struct CodeSources {
  const uint8_t *qc, *kc, *vc;
  int rows_per_head;
  uint64_t v_row_bytes;
};

CodeSources workspace_codes(void* ws, const WsLayout& L) {
  const uint8_t* w = static_cast<const uint8_t*>(ws);
  return CodeSources{w + L.qc, w + L.kc, w + L.vc, L.npad, static_cast<uint64_t>(L.npad) / 2};
}

mxattn_status attend_impl(void* out, int B, int Hq, int Hkv, int N, int d, int causal, int scale_mode, int pnq,
                          int out_dtype, void* ws, cudaStream_t st, const WsLayout& L, const CodeSources& src,
                          int dbg_bh, int dbg_r0, int dbg_r1, uint8_t* p_codes, uint8_t* p_scales,
                          unsigned int* status = nullptr) {
  uint8_t* w = static_cast<uint8_t*>(ws);
  CUtensorMap tq, tk, tv;
  const CUtensorMapSwizzle qk_swz = (d == 128) ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
  const uint64_t rph = static_cast<uint64_t>(src.rows_per_head);
  if (!make_map(&tq, src.qc, d / 2, static_cast<uint64_t>(B) * Hq * rph, d / 2, kTile, qk_swz) ||
      !make_map(&tk, src.kc, d / 2, static_cast<uint64_t>(B) * Hkv * rph, d / 2, kKvTile, qk_swz) ||
      !make_map(&tv, src.vc, src.v_row_bytes, static_cast<uint64_t>(B) * Hkv * d, kKvTile / 2, d,
                CU_TENSOR_MAP_SWIZZLE_64B))
    return MXATTN_ERR_CUDA;
  AttnParams p{};
  p.qsf = w + L.qs;
  p.ksf = w + L.ks;
  p.vsf = w + L.vs;
  p.out = out;
  p.out_bf16 = (out_dtype == MXATTN_OUT_BF16) ? 1 : 0;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = N;
  p.Npad = L.npad;
  p.rows_per_head = src.rows_per_head;
  p.causal = causal ? 1 : 0;
  p.mode = scale_mode;
  p.pnq = pnq;
  p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(d)));
  p.status = status ? status : reinterpret_cast<unsigned int*>(w);
  p.dbg_codes = p_codes;
  p.dbg_scales = p_scales;
  p.dbg_bh = dbg_bh;
  p.dbg_r0 = dbg_r0;
  p.dbg_r1 = dbg_r1;
  return launch_attention(tq, tk, tv, p, d, st) == cudaSuccess ? MXATTN_OK : MXATTN_ERR_CUDA;
}

mxattn_status check_forward_args(const void* q, const void* k, const void* v, const void* out, int B, int Hq,
                                 int Hkv, int N, int d, int scale_mode, int out_dtype, const void* ws,
                                 size_t ws_bytes, WsLayout* L) {
  if (scale_mode != MXATTN_SCALE_OCP && scale_mode != MXATTN_SCALE_UOS && scale_mode != MXATTN_SCALE_NVFP4)
    return MXATTN_ERR_INVALID_ARG;
  if (out_dtype != MXATTN_OUT_F32 && out_dtype != MXATTN_OUT_BF16) return MXATTN_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || N < 1 || Hq % Hkv != 0) return MXATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return MXATTN_ERR_UNSUPPORTED;
  if (!ws_layout(B, Hq, Hkv, N, d, L)) return MXATTN_ERR_UNSUPPORTED;
  if (q && !aligned(q, 16)) return MXATTN_ERR_INVALID_ARG;
  if (k && !aligned(k, 16)) return MXATTN_ERR_INVALID_ARG;
  if (v && !aligned(v, 16)) return MXATTN_ERR_INVALID_ARG;
  if (out && !aligned(out, 16)) return MXATTN_ERR_INVALID_ARG;
  if (!ws || !aligned(ws, 256)) return MXATTN_ERR_INVALID_ARG;
  if (ws_bytes < L->total) return MXATTN_ERR_WORKSPACE;
  return MXATTN_OK;
}

// The rule of the P~ operand (the `pnq` argument): MXATTN_P_CONVENTIONAL, MXATTN_P_PNQ or
// MXATTN_P_EFQ; the exp-free rule is defined for power-of-two (MXFP4) block scales only.
mxattn_status check_p_rule(int pnq, int scale_mode) {
  if (pnq < MXATTN_P_CONVENTIONAL || pnq > MXATTN_P_EFQ) return MXATTN_ERR_INVALID_ARG;
  if (pnq == MXATTN_P_EFQ && scale_mode == MXATTN_SCALE_NVFP4) return MXATTN_ERR_UNSUPPORTED;
  return MXATTN_OK;
}

// GEMM workspace: status area, then the scale atoms of A and B [row tile][kgroup][512].
struct GemmLayout {
  size_t sfa, sfb, total;
  int k_stages, kgroups, tiles_m, tiles_n128;
};

bool gemm_layout(int64_t M, int64_t N, int64_t K, GemmLayout* L, bool nvfp4 = false) {
  if (M < 1 || N < 1 || K < 32 || K % 32 != 0 || N % 8 != 0) return false;
  if (M >= (1ll << 31) || N >= (1ll << 31) || K >= (1ll << 31)) return false;
  if ((M + 127) / 128 > 65535) return false;
  L->k_stages = static_cast<int>((K + 255) / 256);
  L->kgroups = (nvfp4 ? 4 : 2) * L->k_stages;
  L->tiles_m = static_cast<int>((M + 127) / 128);
  L->tiles_n128 = 2 * static_cast<int>((N + 255) / 256);
  size_t off = kAlign;
  L->sfa = off;
  off = align_up(off + static_cast<size_t>(L->tiles_m) * L->kgroups * 512, kAlign);
  L->sfb = off;
  off = align_up(off + static_cast<size_t>(L->tiles_n128) * L->kgroups * 512, kAlign);
  L->total = off;
  return true;
}

}  // namespace

extern "C" {

size_t mxattn_gemm_workspace_size(int64_t M, int64_t N, int64_t K) {
  GemmLayout L;
  return gemm_layout(M, N, K, &L) ? L.total : 0;
}

size_t mxattn_gemm_nvfp4_workspace_size(int64_t M, int64_t N, int64_t K) {
  GemmLayout L;
  return gemm_layout(M, N, K, &L, true) ? L.total : 0;
}

static mxattn_status gemm_impl(const uint8_t* a_codes, const uint8_t* a_scales, const uint8_t* b_codes,
                               const uint8_t* b_scales, void* c, int64_t M, int64_t N, int64_t K, int out_dtype,
                               void* workspace, size_t workspace_bytes, void* stream, bool nvfp4) {
  if (!a_codes || !a_scales || !b_codes || !b_scales || !c || !workspace) return MXATTN_ERR_INVALID_ARG;
  if (out_dtype != MXATTN_OUT_F32 && out_dtype != MXATTN_OUT_BF16) return MXATTN_ERR_INVALID_ARG;
  if (M < 1 || N < 1 || K < 1) return MXATTN_ERR_INVALID_ARG;
  if (!aligned(a_codes, 16) || !aligned(b_codes, 16) || !aligned(c, 16) || !aligned(workspace, 256))
    return MXATTN_ERR_INVALID_ARG;
  GemmLayout L;
  if (!gemm_layout(M, N, K, &L, nvfp4)) return MXATTN_ERR_UNSUPPORTED;
  if (workspace_bytes < L.total) return MXATTN_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* w = static_cast<uint8_t*>(workspace);
  if (cudaMemsetAsync(w, 0, 256, st) != cudaSuccess) return MXATTN_ERR_CUDA;
  const uint32_t kb = static_cast<uint32_t>(K / (nvfp4 ? 16 : 32));   // scale bytes per row
  const ScaleRepackParams reps[2] = {
      {a_scales, w + L.sfa, 1u, static_cast<uint32_t>(L.tiles_m), static_cast<uint32_t>(M), kb, 0,
       static_cast<uint32_t>(L.kgroups)},
      {b_scales, w + L.sfb, 1u, static_cast<uint32_t>(L.tiles_n128), static_cast<uint32_t>(N), kb, 0,
       static_cast<uint32_t>(L.kgroups)}};
  for (const ScaleRepackParams& r : reps)
    if (launch_repack_scales(r, st) != cudaSuccess) return MXATTN_ERR_CUDA;
  CUtensorMap ta, tb, tc;
  if (!make_map(&ta, a_codes, static_cast<uint64_t>(K / 2), static_cast<uint64_t>(M), 128, 128,
                CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&tb, b_codes, static_cast<uint64_t>(K / 2), static_cast<uint64_t>(N), 128, 256,
                CU_TENSOR_MAP_SWIZZLE_128B))
    return MXATTN_ERR_CUDA;
  if (out_dtype == MXATTN_OUT_BF16) {
    // C as [M, N] bf16 for the epilogue's TMA stores: 128 rows x 64 columns per box, 128B swizzle
    if (!make_map_typed(&tc, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, c, static_cast<uint64_t>(N), static_cast<uint64_t>(M),
                        static_cast<uint64_t>(N) * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B))
      return MXATTN_ERR_CUDA;
  } else {
    std::memset(&tc, 0, sizeof(tc));   // fp32 output is stored without TMA
  }
  GemmParams p{};
  p.sfa = w + L.sfa;
  p.sfb = w + L.sfb;
  p.c = c;
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.k_stages = L.k_stages;
  p.kgroups = L.kgroups;
  p.out_bf16 = (out_dtype == MXATTN_OUT_BF16) ? 1 : 0;
  p.nvfp4 = nvfp4 ? 1 : 0;
  p.status = reinterpret_cast<unsigned int*>(w);
  return launch_gemm(ta, tb, tc, p, st) == cudaSuccess ? MXATTN_OK : MXATTN_ERR_CUDA;
}

mxattn_status mxattn_gemm(const uint8_t* a_codes, const uint8_t* a_scales, const uint8_t* b_codes,
                          const uint8_t* b_scales, void* c, int64_t M, int64_t N, int64_t K, int out_dtype,
                          void* workspace, size_t workspace_bytes, void* stream) {
  return gemm_impl(a_codes, a_scales, b_codes, b_scales, c, M, N, K, out_dtype, workspace, workspace_bytes, stream,
                   false);
}

mxattn_status mxattn_gemm_nvfp4(const uint8_t* a_codes, const uint8_t* a_scales, const uint8_t* b_codes,
                                const uint8_t* b_scales, void* c, int64_t M, int64_t N, int64_t K, int out_dtype,
                                void* workspace, size_t workspace_bytes, void* stream) {
  return gemm_impl(a_codes, a_scales, b_codes, b_scales, c, M, N, K, out_dtype, workspace, workspace_bytes, stream,
                   true);
}

mxattn_status mxattn_quantize_nvfp4(const void* x, int64_t rows, int64_t cols, uint8_t* codes, uint8_t* scales,
                                    void* stream) {
  if (rows < 0 || cols < 0) return MXATTN_ERR_INVALID_ARG;
  if (rows == 0 || cols == 0) return MXATTN_OK;
  if (!x || !codes || !scales) return MXATTN_ERR_INVALID_ARG;
  if (!aligned(x, 2) || !aligned(codes, 8)) return MXATTN_ERR_INVALID_ARG;
  if (rows >= (1ll << 31) || cols >= (1ll << 31) || static_cast<uint64_t>(rows) * ((cols + 15) / 16) >= (1ull << 40))
    return MXATTN_ERR_UNSUPPORTED;
  NvQuantParams p{};
  p.x = static_cast<const __nv_bfloat16*>(x);
  p.heads = 1;
  p.rows = static_cast<uint32_t>(rows);
  p.cols = static_cast<uint32_t>(cols);
  p.codes = codes;
  p.scales = scales;
  p.vec_ok = (aligned(x, 16) && cols % 8 == 0) ? 1 : 0;
  return launch_quantize_rows_nvfp4(p, static_cast<cudaStream_t>(stream)) == cudaSuccess ? MXATTN_OK
                                                                                          : MXATTN_ERR_CUDA;
}


int mxattn_version(void) { return 102; }

const char* mxattn_status_string(int status) {
  switch (status) {
    case MXATTN_OK: return "ok";
    case MXATTN_ERR_INVALID_ARG: return "invalid argument";
    case MXATTN_ERR_UNSUPPORTED: return "unsupported shape or option";
    case MXATTN_ERR_WORKSPACE: return "workspace too small";
    case MXATTN_ERR_CUDA: return "CUDA error";
    case MXATTN_ERR_TIMEOUT: return "device pipeline timeout";
    default: return "unknown status";
  }
}

mxattn_status mxattn_quantize(const void* x, int64_t batch, int64_t rows, int64_t cols, int transpose,
                              int scale_mode, uint8_t* codes, uint8_t* scales, void* stream) {
  if (batch < 0 || rows < 0 || cols < 0) return MXATTN_ERR_INVALID_ARG;
  if (scale_mode != MXATTN_SCALE_OCP && scale_mode != MXATTN_SCALE_UOS) return MXATTN_ERR_INVALID_ARG;
  if (transpose != 0 && transpose != 1) return MXATTN_ERR_INVALID_ARG;
  if (batch == 0 || rows == 0 || cols == 0) return MXATTN_OK;
  if (!x || !codes || !scales) return MXATTN_ERR_INVALID_ARG;
  if (!aligned(x, 2) || !aligned(codes, 16)) return MXATTN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int vec_ok = (aligned(x, 16) && cols % 8 == 0) ? 1 : 0;
  if (transpose == 0) {
    const uint64_t kb = (static_cast<uint64_t>(cols) + 31) / 32;
    if (static_cast<uint64_t>(batch) * rows * kb >= (1ull << 31) || rows >= (1ll << 31) || cols >= (1ll << 31))
      return MXATTN_ERR_UNSUPPORTED;
    RowQuantParams p{};
    p.x = static_cast<const __nv_bfloat16*>(x);
    p.heads = static_cast<uint32_t>(batch);
    p.rows = static_cast<uint32_t>(rows);
    p.rows_pad = static_cast<uint32_t>(rows);
    p.cols = static_cast<uint32_t>(cols);
    p.kb = static_cast<uint32_t>(kb);
    p.codes = codes;
    p.scales = scales;
    p.mode = scale_mode;
    p.sf_layout = kSfRowMajor;
    p.vec_ok = vec_ok;
    return launch_quantize_rows(p, st) == cudaSuccess ? MXATTN_OK : MXATTN_ERR_CUDA;
  }
  const uint64_t nblk = (static_cast<uint64_t>(rows) + 31) / 32;
  if (batch > 65535 || static_cast<uint64_t>(batch) * cols * nblk >= (1ull << 31) || rows >= (1ll << 31) ||
      cols >= (1ll << 31))
    return MXATTN_ERR_UNSUPPORTED;
  ColQuantParams p{};
  p.x = static_cast<const __nv_bfloat16*>(x);
  p.heads = static_cast<uint32_t>(batch);
  p.rows = static_cast<uint32_t>(rows);
  p.cols = static_cast<uint32_t>(cols);
  p.nblk = static_cast<uint32_t>(nblk);
  p.codes = codes;
  p.scales = scales;
  p.mode = scale_mode;
  p.sf_layout = kSfRowMajor;
  p.vec_ok = vec_ok;
  return launch_quantize_cols(p, st) == cudaSuccess ? MXATTN_OK : MXATTN_ERR_CUDA;
}

size_t mxattn_forward_workspace_size(int B, int Hq, int Hkv, int N, int d) {
  WsLayout L;
  return ws_layout(B, Hq, Hkv, N, d, &L) ? L.total : 0;
}

mxattn_status mxattn_forward_prepare(const void* q, const void* k, const void* v, int B, int Hq, int Hkv, int N,
                                     int d, int scale_mode, void* workspace, size_t workspace_bytes,
                                     void* stream) {
  if (!q || !k || !v) return MXATTN_ERR_INVALID_ARG;
  WsLayout L;
  mxattn_status s = check_forward_args(q, k, v, nullptr, B, Hq, Hkv, N, d, scale_mode, MXATTN_OUT_F32, workspace,
                                       workspace_bytes, &L);
  if (s != MXATTN_OK) return s;
  if (cudaMemsetAsync(workspace, 0, 256, static_cast<cudaStream_t>(stream)) != cudaSuccess) return MXATTN_ERR_CUDA;
  return prepare_impl(q, k, v, B, Hq, Hkv, N, d, scale_mode, workspace, workspace_bytes,
                      static_cast<cudaStream_t>(stream), L);
}

mxattn_status mxattn_forward_attend(void* out, int B, int Hq, int Hkv, int N, int d, int causal, int scale_mode,
                                    int pnq, int out_dtype, void* workspace, size_t workspace_bytes,
                                    void* stream) {
  if (!out) return MXATTN_ERR_INVALID_ARG;
  WsLayout L;
  mxattn_status s = check_forward_args(nullptr, nullptr, nullptr, out, B, Hq, Hkv, N, d, scale_mode, out_dtype,
                                       workspace, workspace_bytes, &L);
  if (s == MXATTN_OK) s = check_p_rule(pnq, scale_mode);
  if (s != MXATTN_OK) return s;
  return attend_impl(out, B, Hq, Hkv, N, d, causal, scale_mode, pnq, out_dtype, workspace,
                     static_cast<cudaStream_t>(stream), L, workspace_codes(workspace, L), -1, 0, 0, nullptr,
                     nullptr);
}

mxattn_status mxattn_forward_quantized(const uint8_t* qc, const uint8_t* qs, const uint8_t* kc, const uint8_t* ks,
                                       const uint8_t* vtc, const uint8_t* vts, void* out, int B, int Hq, int Hkv,
                                       int N, int d, int causal, int p_scale_mode, int pnq, int out_dtype,
                                       void* workspace, size_t workspace_bytes, void* stream) {
  if (!qc || !qs || !kc || !ks || !vtc || !vts || !out) return MXATTN_ERR_INVALID_ARG;
  if (!aligned(qc, 16) || !aligned(kc, 16) || !aligned(vtc, 16)) return MXATTN_ERR_INVALID_ARG;
  WsLayout L;
  mxattn_status s = check_forward_args(nullptr, nullptr, nullptr, out, B, Hq, Hkv, N, d, p_scale_mode, out_dtype,
                                       workspace, workspace_bytes, &L);
  if (s == MXATTN_OK) s = check_p_rule(pnq, p_scale_mode);
  if (s != MXATTN_OK) return s;
  if (p_scale_mode == MXATTN_SCALE_NVFP4) return MXATTN_ERR_UNSUPPORTED;   // MXFP4 operands only
  if (static_cast<uint64_t>(B) * Hq * N >= (1ull << 31)) return MXATTN_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* w = static_cast<uint8_t*>(workspace);
  if (cudaMemsetAsync(w, 0, 256, st) != cudaSuccess) return MXATTN_ERR_CUDA;
  const uint32_t tiles = static_cast<uint32_t>(L.npad / kTile);
  const uint32_t nblk = static_cast<uint32_t>((N + 31) / 32);
  const ScaleRepackParams reps[3] = {
      {qs, w + L.qs, static_cast<uint32_t>(B * Hq), tiles, static_cast<uint32_t>(N), static_cast<uint32_t>(d / 32), 0},
      {ks, w + L.ks, static_cast<uint32_t>(B * Hkv), tiles, static_cast<uint32_t>(N), static_cast<uint32_t>(d / 32), 0},
      {vts, w + L.vs, static_cast<uint32_t>(B * Hkv), tiles, static_cast<uint32_t>(d), nblk, 1}};
  for (const ScaleRepackParams& r : reps)
    if (launch_repack_scales(r, st) != cudaSuccess) return MXATTN_ERR_CUDA;
  const CodeSources src{qc, kc, vtc, N, static_cast<uint64_t>(nblk) * 16};
  return attend_impl(out, B, Hq, Hkv, N, d, causal, p_scale_mode, pnq, out_dtype, workspace, st, L, src, -1, 0, 0,
                     nullptr, nullptr);
}

mxattn_status mxattn_forward(const void* q, const void* k, const void* v, void* out, int B, int Hq, int Hkv,
                             int N, int d, int causal, int scale_mode, int pnq, int out_dtype, void* workspace,
                             size_t workspace_bytes, void* stream) {
  return mxattn_forward_debug(q, k, v, out, B, Hq, Hkv, N, d, causal, scale_mode, pnq, out_dtype, workspace,
                              workspace_bytes, stream, -1, 0, 0, nullptr, nullptr);
}

mxattn_status mxattn_forward_debug(const void* q, const void* k, const void* v, void* out, int B, int Hq,
                                   int Hkv, int N, int d, int causal, int scale_mode, int pnq, int out_dtype,
                                   void* workspace, size_t workspace_bytes, void* stream, int dbg_bh, int dbg_r0,
                                   int dbg_r1, uint8_t* p_codes, uint8_t* p_scales) {
  if (!q || !k || !v || !out) return MXATTN_ERR_INVALID_ARG;
  WsLayout L;
  mxattn_status s = check_forward_args(q, k, v, out, B, Hq, Hkv, N, d, scale_mode, out_dtype, workspace,
                                       workspace_bytes, &L);
  if (s == MXATTN_OK) s = check_p_rule(pnq, scale_mode);
  if (s != MXATTN_OK) return s;
  if (p_codes || p_scales) {
    if (!p_codes || !p_scales || dbg_bh < 0 || dbg_bh >= B * Hq || dbg_r0 < 0 || dbg_r1 <= dbg_r0 ||
        dbg_r1 > L.npad || !aligned(p_codes, 16) || !aligned(p_scales, 4))
      return MXATTN_ERR_INVALID_ARG;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(workspace, 0, 256, st) != cudaSuccess) return MXATTN_ERR_CUDA;
  s = prepare_impl(q, k, v, B, Hq, Hkv, N, d, scale_mode, workspace, workspace_bytes, st, L);
  if (s != MXATTN_OK) return s;
  return attend_impl(out, B, Hq, Hkv, N, d, causal, scale_mode, pnq, out_dtype, workspace, st, L,
                     workspace_codes(workspace, L), dbg_bh, dbg_r0, dbg_r1, p_codes, p_scales);
}

// ---------------------------------------------------------------- host-buffer pipeline
// mxattn_forward on host buffers: KV-head groups ("chunks") flow through kHostSlots device slots.
// Per chunk, the inputs are copied in on one stream, quantized and attended on one of two compute
// streams (the caller's and a side stream, alternating by chunk), and the output is copied out on
// a fourth. Each part of a slot is reused as soon as its last reader is done: the bf16 inputs once
// the quantizers have read them, the codes once the attention kernel has, the output once it has
// been copied out. So the host-to-device stream runs back to back while the device-to-host copies
// go the other way, and the attention kernel of one chunk fills the SMs that the tail of the
// previous chunk's kernel leaves idle. Heads are independent, so the result equals mxattn_forward's.

constexpr int kHostSlots = 3;          // device slots the chunks rotate through
constexpr long kHostChunkCtas = 512;   // attention CTAs per chunk (rounded up to whole KV heads)

struct HostPlan {
  int cg;                  // KV heads per chunk (the slots are sized for it)
  std::vector<int> sizes;  // KV heads per chunk, in order
  size_t q_bytes, kv_bytes, out_bytes, attn_ws;   // per slot, for a full chunk
  size_t slot_bytes, total;
};

static bool host_plan(int B, int Hq, int Hkv, int N, int d, int out_dtype, HostPlan* P) {
  WsLayout L;
  if (!ws_layout(B, Hq, Hkv, N, d, &L)) return false;
  if (out_dtype != MXATTN_OUT_F32 && out_dtype != MXATTN_OUT_BF16) return false;
  const int group = Hq / Hkv;
  const int units = B * Hkv;
  const long n_qt = (N + kTile - 1) / kTile;
  // small chunks keep the pipeline's fill (the first chunk's copy-in) and drain (the last chunk's
  // kernel and copy-out) short; the wave tail of each chunk's kernel is filled by the next chunk's
  // kernel on the other compute stream
  const long target_ctas = kHostChunkCtas;
  long cg = (target_ctas + group * n_qt - 1) / (group * n_qt);
  if (cg < 1) cg = 1;
  if (cg > units) cg = units;
  P->cg = static_cast<int>(cg);
  // full chunks, except that the first and the last hold half a chunk when there are more than
  // two: a shorter first copy-in and a shorter last kernel and copy-out trim the fill and the
  // drain (1% on the video-DiT shape)
  P->sizes.clear();
  const int full = static_cast<int>(cg);
  const int edge = units > 2 * full ? (full > 1 ? full / 2 : 1) : 0;
  if (edge) P->sizes.push_back(edge);
  for (int u = edge; u < units - edge; u += full) P->sizes.push_back(std::min(full, units - edge - u));
  if (edge) P->sizes.push_back(edge);
  const size_t hd = static_cast<size_t>(N) * d;
  P->q_bytes = static_cast<size_t>(cg) * group * hd * 2;
  P->kv_bytes = static_cast<size_t>(cg) * hd * 2;
  P->out_bytes = static_cast<size_t>(cg) * group * hd * (out_dtype == MXATTN_OUT_F32 ? 4 : 2);
  WsLayout Lc;
  if (!ws_layout(1, static_cast<int>(cg) * group, static_cast<int>(cg), N, d, &Lc)) return false;
  P->attn_ws = Lc.total;
  P->slot_bytes = align_up(P->q_bytes, kAlign) + 2 * align_up(P->kv_bytes, kAlign) + align_up(P->out_bytes, kAlign) +
                  align_up(P->attn_ws, kAlign);
  P->total = kAlign + kHostSlots * P->slot_bytes;
  return true;
}

struct SideStreams {
  cudaStream_t in = nullptr, out = nullptr, comp = nullptr;
};

static mxattn_status side_streams(SideStreams* out) {
  static std::mutex mu;
  static SideStreams cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MXATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  SideStreams& c = cache[dev];
  if (!c.in && cudaStreamCreateWithFlags(&c.in, cudaStreamNonBlocking) != cudaSuccess) return MXATTN_ERR_CUDA;
  if (!c.out && cudaStreamCreateWithFlags(&c.out, cudaStreamNonBlocking) != cudaSuccess) return MXATTN_ERR_CUDA;
  if (!c.comp && cudaStreamCreateWithFlags(&c.comp, cudaStreamNonBlocking) != cudaSuccess) return MXATTN_ERR_CUDA;
  *out = c;
  return MXATTN_OK;
}

size_t mxattn_forward_host_workspace_size(int B, int Hq, int Hkv, int N, int d, int out_dtype) {
  HostPlan P;
  return host_plan(B, Hq, Hkv, N, d, out_dtype, &P) ? P.total : 0;
}

mxattn_status mxattn_forward_host(const void* q, const void* k, const void* v, void* out, int B, int Hq, int Hkv,
                                  int N, int d, int causal, int scale_mode, int pnq, int out_dtype, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !out) return MXATTN_ERR_INVALID_ARG;
  WsLayout L;
  mxattn_status s = check_forward_args(nullptr, nullptr, nullptr, nullptr, B, Hq, Hkv, N, d, scale_mode, out_dtype,
                                       workspace, workspace_bytes, &L);
  if (s != MXATTN_OK && s != MXATTN_ERR_WORKSPACE) return s;
  if ((s = check_p_rule(pnq, scale_mode)) != MXATTN_OK) return s;
  HostPlan P;
  if (!host_plan(B, Hq, Hkv, N, d, out_dtype, &P)) return MXATTN_ERR_UNSUPPORTED;
  if (workspace_bytes < P.total) return MXATTN_ERR_WORKSPACE;
  SideStreams ss;
  if ((s = side_streams(&ss)) != MXATTN_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* w = static_cast<uint8_t*>(workspace);
  unsigned int* status = reinterpret_cast<unsigned int*>(w);
  const int group = Hq / Hkv;
  const size_t hd = static_cast<size_t>(N) * d;
  const size_t out_elem = (out_dtype == MXATTN_OUT_F32) ? 4 : 2;

  // events: start (orders the side streams after earlier work on the caller's stream); per chunk
  // inputs-in, inputs-consumed, compute-done, output-out; and one tail per side stream
  const int chunks = static_cast<int>(P.sizes.size());
  std::vector<cudaEvent_t> ev(4 + 4 * static_cast<size_t>(chunks), nullptr);
  for (auto& e : ev)
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) s = MXATTN_ERR_CUDA;
  auto ev_in = [&](int c) { return ev[1 + 4 * c]; };
  auto ev_prep = [&](int c) { return ev[2 + 4 * c]; };
  auto ev_comp = [&](int c) { return ev[3 + 4 * c]; };
  auto ev_out = [&](int c) { return ev[4 + 4 * c]; };
  auto ok = [&](cudaError_t e) { if (e != cudaSuccess && s == MXATTN_OK) s = MXATTN_ERR_CUDA; };
  if (s == MXATTN_OK) {
    ok(cudaMemsetAsync(w, 0, 256, st));
    ok(cudaEventRecord(ev[0], st));
    ok(cudaStreamWaitEvent(ss.in, ev[0], 0));
    ok(cudaStreamWaitEvent(ss.out, ev[0], 0));
    ok(cudaStreamWaitEvent(ss.comp, ev[0], 0));
  }
  int u0 = 0;
  for (int c = 0; c < chunks && s == MXATTN_OK; u0 += P.sizes[c], ++c) {
    const int cu = P.sizes[c];                                   // KV heads in this chunk
    const bool reuse = c >= kHostSlots;                          // the slot held chunk c - kHostSlots
    cudaStream_t cs = (c & 1) ? ss.comp : st;
    uint8_t* slot = w + kAlign + static_cast<size_t>(c % kHostSlots) * P.slot_bytes;
    uint8_t* dq = slot;
    uint8_t* dk = dq + align_up(P.q_bytes, kAlign);
    uint8_t* dv = dk + align_up(P.kv_bytes, kAlign);
    uint8_t* dout = dv + align_up(P.kv_bytes, kAlign);
    uint8_t* aws = dout + align_up(P.out_bytes, kAlign);
    const size_t qb = static_cast<size_t>(cu) * group * hd * 2, kvb = static_cast<size_t>(cu) * hd * 2;
    const size_t ob = static_cast<size_t>(cu) * group * hd * out_elem;
    const size_t q_off = static_cast<size_t>(u0) * group * hd, kv_off = static_cast<size_t>(u0) * hd;
    // inputs, once the quantizers of the slot's previous chunk have read its bf16 buffers
    if (reuse) ok(cudaStreamWaitEvent(ss.in, ev_prep(c - kHostSlots), 0));
    ok(cudaMemcpyAsync(dq, static_cast<const uint8_t*>(q) + q_off * 2, qb, cudaMemcpyHostToDevice, ss.in));
    ok(cudaMemcpyAsync(dk, static_cast<const uint8_t*>(k) + kv_off * 2, kvb, cudaMemcpyHostToDevice, ss.in));
    ok(cudaMemcpyAsync(dv, static_cast<const uint8_t*>(v) + kv_off * 2, kvb, cudaMemcpyHostToDevice, ss.in));
    ok(cudaEventRecord(ev_in(c), ss.in));
    // quantizers: the codes region is free once the previous chunk's attention kernel has read it
    ok(cudaStreamWaitEvent(cs, ev_in(c), 0));
    if (reuse) ok(cudaStreamWaitEvent(cs, ev_comp(c - kHostSlots), 0));
    WsLayout Lc;
    ws_layout(1, cu * group, cu, N, d, &Lc);
    if (s == MXATTN_OK) s = prepare_impl(dq, dk, dv, 1, cu * group, cu, N, d, scale_mode, aws, P.attn_ws, cs, Lc);
    ok(cudaEventRecord(ev_prep(c), cs));
    // attention: the output buffer is free once the previous chunk's output has been copied out
    if (reuse) ok(cudaStreamWaitEvent(cs, ev_out(c - kHostSlots), 0));
    if (s == MXATTN_OK)
      s = attend_impl(dout, 1, cu * group, cu, N, d, causal, scale_mode, pnq, out_dtype, aws, cs, Lc,
                      workspace_codes(aws, Lc), -1, 0, 0, nullptr, nullptr, status);
    ok(cudaEventRecord(ev_comp(c), cs));
    // output
    ok(cudaStreamWaitEvent(ss.out, ev_comp(c), 0));
    ok(cudaMemcpyAsync(static_cast<uint8_t*>(out) + q_off * out_elem, dout, ob, cudaMemcpyDeviceToHost, ss.out));
    ok(cudaEventRecord(ev_out(c), ss.out));
  }
  // the call completes on the caller's stream once everything it queued on the side streams has
  // run, on an error path too, so that the caller may free the buffers once its stream is done
  cudaStream_t side[3] = {ss.in, ss.comp, ss.out};
  for (int i = 0; i < 3; ++i) {
    cudaEvent_t tail = ev[1 + 4 * static_cast<size_t>(chunks) + i];
    if (tail && cudaEventRecord(tail, side[i]) == cudaSuccess) ok(cudaStreamWaitEvent(st, tail, 0));
    else if (s == MXATTN_OK) s = MXATTN_ERR_CUDA;
  }
  for (auto& e : ev)
    if (e) cudaEventDestroy(e);   // released once recorded work completes
  return s;
}

mxattn_status mxattn_selftest_wait_timeout(void* workspace, void* stream) {
  if (!workspace || !aligned(workspace, 256)) return MXATTN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned int* w = static_cast<unsigned int*>(workspace);
  if (cudaMemsetAsync(w, 0, 256, st) != cudaSuccess) return MXATTN_ERR_CUDA;
  return launch_wait_timeout_selftest(w, w + 1, st) == cudaSuccess ? MXATTN_OK : MXATTN_ERR_CUDA;
}

mxattn_status mxattn_check_status(void* workspace, void* stream, unsigned int* detail) {
  if (!workspace) return MXATTN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned int word = 0;
  if (cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return MXATTN_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return MXATTN_ERR_CUDA;
  if (detail) *detail = word;
  if (word != 0) {
    if (cudaMemsetAsync(workspace, 0, sizeof(word), st) != cudaSuccess) return MXATTN_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return MXATTN_ERR_CUDA;
    return MXATTN_ERR_TIMEOUT;
  }
  return MXATTN_OK;
}

}  // extern "C"

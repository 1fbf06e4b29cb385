// MXFP4 attention forward for sm_100a: block-scaled FP4 tensor-core contractions inside a
// FlashAttention-style online-softmax loop, with Pre-Normalization Quantization of P~.
//
// Method (MXAttention abstract; EFQ-Softmax abstract for the unchanged FlashAttention loop):
//   S_j  = dq(Q) dq(K_j)^T                    tcgen05.mma kind::mxf4, UE8M0 scales, fp32 in TMEM
//   m'   = max(m, rowmax S_j);  alpha = 2^((m - m') * c),  c = log2(e) / sqrt(d)
//   P~_j = 2^((S_j - m') * c)                  the unnormalised exponentials
//   PNQ:  P~_j is quantized to MXFP4 along keys (32-key blocks, OCP or UOS exponent) BEFORE any
//         row sum; the same dequantized operand feeds
//           O = alpha * O + dq(P~_j) dq(V_j)    (numerator, tcgen05.mma kind::mxf4)
//           l = alpha * l + dq(P~_j) 1          (denominator: the same block-scaled MMA against a
//                                                constant ones operand, N = 16, column 0)
//   pnq = 0 keeps the conventional path: l sums the unquantized fp32 P~ on the CUDA cores.
//   out = O / l.
//
// One CTA owns one 128-query tile of one (batch, query head); keys are visited in tiles of 128
// in increasing order (P~ codes depend on the running max in force, so the order is part of
// the definition). Warp roles (256 threads):
//   warp 0     TMA producer: Q tile once, then K / V^T tiles and their scale atoms into a
//              NSTAGE-deep shared-memory ring (mbarrier complete_tx).
//   warp 1     TMEM owner and MMA issuer (one elected thread): copies scale atoms to TMEM with
//              tcgen05.cp, issues S = QK^T into one of two S buffers and O += P~ V^T.
//   warps 4-7  softmax warpgroup, one thread per query row (TMEM lane = row): reads S with
//              tcgen05.ld, updates the running max, computes P~, quantizes it in registers,
//              writes codes (64B-swizzled, the MMA operand layout) and scale atoms to shared
//              memory, keeps the row sum, rescales O in TMEM when the max moves, and finally
//              normalises and stores the output.
// TMEM (512 columns): S0 [0,128) S1 [128,256) O [256,256+d) row sum L [384,400), scale atoms at
// 400..419 (Q, K, V, P~, ones).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "mxattn_internal.h"
#include "sm100_ptx.cuh"

namespace mxattn {

constexpr int kBM = 128;          // query rows per CTA
constexpr int kBN = 128;          // keys per KV tile
constexpr int kThreads = 256;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256, kColL = 384;
constexpr uint32_t kColSfQ = 400, kColSfK = 404, kColSfV = 408, kColSfP = 412, kColSf1 = 416;
constexpr int kOnesRows = 16;     // N of the row-sum MMA: row 0 all ones, rows 1..15 zero
constexpr size_t kMinSmem = 120 * 1024;   // keeps one CTA per SM (its TMEM allocation is 512)

template <int D>
struct Cfg {
  static constexpr int kStages = 6;
  static constexpr int kQRowBytes = D / 2;                 // packed E2M1 per Q/K row
  static constexpr int kQTileBytes = kBM * kQRowBytes;
  static constexpr int kKTileBytes = kBN * kQRowBytes;
  static constexpr int kVTileBytes = D * (kBN / 2);        // V^T: D rows of 128 keys
  static constexpr int kPTileBytes = kBM * (kBN / 2);
  static constexpr uint32_t kQKLayout = (D == 128) ? kLayoutSw64 : kLayoutSw32;
  static constexpr uint32_t kQKSbo = 8 * kQRowBytes;       // 8-row swizzle atom
};

template <int D>
struct __align__(1024) Smem {
  uint8_t q[Cfg<D>::kQTileBytes];
  uint8_t k[Cfg<D>::kStages][Cfg<D>::kKTileBytes];
  uint8_t v[Cfg<D>::kStages][Cfg<D>::kVTileBytes];
  uint8_t p[Cfg<D>::kPTileBytes];
  uint8_t ones[kOnesRows * (kBN / 2)];
  uint8_t qsf[512];
  uint8_t ksf[Cfg<D>::kStages][512];
  uint8_t vsf[Cfg<D>::kStages][512];
  uint8_t psf[512];
  uint8_t onesf[512];
  uint64_t bar_q;
  uint64_t bar_kv_full[Cfg<D>::kStages];
  uint64_t bar_kv_empty[Cfg<D>::kStages];
  uint64_t bar_s_full[2];
  uint64_t bar_s_empty[2];
  uint64_t bar_p_full;
  uint64_t bar_pv_done;
  uint64_t bar_drain;
  uint32_t tmem_base;
  int abort_flag;
};

template <int D>
constexpr size_t smem_bytes() {
  return (sizeof(Smem<D>) + 1024 > kMinSmem) ? sizeof(Smem<D>) + 1024 : kMinSmem;
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float ex2_approx_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Bounded wait that ignores the abort flag (used only to drain in-flight copies / MMAs).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > 200ull * 1000ull * 1000ull) break;
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    mxattn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using C = Cfg<D>;
  constexpr int NS = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  Smem<D>& s = *reinterpret_cast<Smem<D>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work tile: (b, kv head g, query head within group, q tile); q tile fastest so that
  //      co-resident CTAs share one KV head in L2; causal runs the longest tiles first.
  const int n_qt = p.Npad / kBM;
  const int group = p.Hq / p.Hkv;
  int idx = blockIdx.x;
  int qt = idx % n_qt;
  idx /= n_qt;
  const int bh_q = idx;                       // b * Hq + h  (h = g * group + hh)
  const int b = idx / p.Hq;
  const int h = idx % p.Hq;
  const int bh_kv = b * p.Hkv + h / group;
  if (p.causal) qt = n_qt - 1 - qt;
  const int n_kv_all = p.Npad / kBN;
  const int n_kv = p.causal ? min(qt + 1, n_kv_all) : n_kv_all;

  if (threadIdx.x == 0) {
    mbar_init(&s.bar_q, 1);
    for (int i = 0; i < NS; ++i) {
      mbar_init(&s.bar_kv_full[i], 1);
      mbar_init(&s.bar_kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.bar_s_full[i], 1);
      mbar_init(&s.bar_s_empty[i], 128);
    }
    mbar_init(&s.bar_p_full, 128);
    mbar_init(&s.bar_pv_done, 1);
    mbar_init(&s.bar_drain, 1);
    s.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&s.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  volatile int* abort_flag = &s.abort_flag;

  if (warp == 0) {
    // ============================ TMA producer ============================
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      mbar_arrive_expect_tx(&s.bar_q, C::kQTileBytes + 512);
      tma_load_2d(s.q, &tmQ, &s.bar_q, 0, bh_q * p.Npad + qt * kBM);
      bulk_load(s.qsf, p.qsf + (static_cast<size_t>(bh_q) * n_qt + qt) * 512, 512, &s.bar_q);
      int issued = 0;
      for (int j = 0; j < n_kv; ++j) {
        const int st = j % NS;
        if (j >= NS) {
          if (!mbar_wait(&s.bar_kv_empty[st], ((j / NS) & 1) ^ 1, abort_flag, p.status,
                         kStatusTimeoutEmpty | st))
            break;
        }
        mbar_arrive_expect_tx(&s.bar_kv_full[st], C::kKTileBytes + C::kVTileBytes + 1024);
        tma_load_2d(s.k[st], &tmK, &s.bar_kv_full[st], 0, bh_kv * p.Npad + j * kBN);
        tma_load_2d(s.v[st], &tmV, &s.bar_kv_full[st], j * (kBN / 2), bh_kv * D);
        const size_t atom = (static_cast<size_t>(bh_kv) * n_kv_all + j) * 512;
        bulk_load(s.ksf[st], p.ksf + atom, 512, &s.bar_kv_full[st]);
        bulk_load(s.vsf[st], p.vsf + atom, 512, &s.bar_kv_full[st]);
        issued = j + 1;
      }
      if (*abort_flag) {
        // let every copy this thread started land before the CTA can exit
        drain_wait(&s.bar_q, 0);
        for (int j = (issued > NS ? issued - NS : 0); j < issued; ++j)
          drain_wait(&s.bar_kv_full[j % NS], (j / NS) & 1);
      }
    }
  } else if (warp == 1) {
    // ============================ MMA issuer ============================
    if (lane == 0) {
      const uint64_t sf_desc_base = smem_desc(0, 0, 128, kLayoutNone);
      auto sf_desc = [&](const void* ptr) { return sf_desc_base | ((smem_u32(ptr) >> 4) & 0x3FFFu); };
      if (p.pnq) {
        // ones operand (row 0 = code 1.0 for every key, rows 1..15 = 0) with unit scales
        uint32_t* ow = reinterpret_cast<uint32_t*>(s.ones);
        for (int i = 0; i < kOnesRows * (kBN / 2) / 4; ++i) ow[i] = (i < (kBN / 2) / 4) ? 0x22222222u : 0u;
        uint32_t* sw = reinterpret_cast<uint32_t*>(s.onesf);
        for (int i = 0; i < 512 / 4; ++i) sw[i] = 0x7F7F7F7Fu;
        fence_proxy_async_smem();
      }
      bool ok = mbar_wait(&s.bar_q, 0, abort_flag, p.status, kStatusTimeoutQ);
      if (ok) {
        tc_fence_after();
        tc_cp_sf(tmem + kColSfQ, sf_desc(s.qsf));
        if (p.pnq) tc_cp_sf(tmem + kColSf1, sf_desc(s.onesf));
      }
      auto issue_s = [&](int j) -> bool {
        const int st = j % NS;
        const int sb = j & 1;
        if (!mbar_wait(&s.bar_kv_full[st], (j / NS) & 1, abort_flag, p.status, kStatusTimeoutKV | st))
          return false;
        if (j >= 2 && !mbar_wait(&s.bar_s_empty[sb], ((j >> 1) - 1) & 1, abort_flag, p.status,
                                 kStatusTimeoutS | sb))
          return false;
        tc_fence_after();
        tc_cp_sf(tmem + kColSfK, sf_desc(s.ksf[st]));
        const uint32_t qa = smem_u32(s.q), ka = smem_u32(s.k[st]);
#pragma unroll
        for (int kk = 0; kk < D / 64; ++kk) {
          const uint64_t ad = smem_desc(qa + kk * 32, 0, C::kQKSbo, C::kQKLayout);
          const uint64_t bd = smem_desc(ka + kk * 32, 0, C::kQKSbo, C::kQKLayout);
          tc_mma_mxf4(tmem + (sb ? kColS1 : kColS0), ad, bd, idesc_mxf4(kBN, 2 * kk, 2 * kk),
                      tmem + kColSfQ, tmem + kColSfK, kk > 0);
        }
        tc_commit(&s.bar_s_full[sb]);
        return true;
      };
      auto issue_pv = [&](int j) -> bool {
        const int st = j % NS;
        if (!mbar_wait(&s.bar_p_full, j & 1, abort_flag, p.status, kStatusTimeoutP)) return false;
        tc_fence_after();
        tc_cp_sf(tmem + kColSfP, sf_desc(s.psf));
        tc_cp_sf(tmem + kColSfV, sf_desc(s.vsf[st]));
        const uint32_t pa = smem_u32(s.p), va = smem_u32(s.v[st]);
#pragma unroll
        for (int kk = 0; kk < kBN / 64; ++kk) {
          const uint64_t ad = smem_desc(pa + kk * 32, 0, 512, kLayoutSw64);
          const uint64_t bd = smem_desc(va + kk * 32, 0, 512, kLayoutSw64);
          tc_mma_mxf4(tmem + kColO, ad, bd, idesc_mxf4(D, 2 * kk, 2 * kk), tmem + kColSfP, tmem + kColSfV,
                      (j > 0 || kk > 0) ? 1u : 0u);
        }
        if (p.pnq) {
          const uint32_t oa = smem_u32(s.ones);
#pragma unroll
          for (int kk = 0; kk < kBN / 64; ++kk) {
            const uint64_t ad = smem_desc(pa + kk * 32, 0, 512, kLayoutSw64);
            const uint64_t bd = smem_desc(oa + kk * 32, 0, 512, kLayoutSw64);
            tc_mma_mxf4(tmem + kColL, ad, bd, idesc_mxf4(kOnesRows, 2 * kk, 2 * kk), tmem + kColSfP,
                        tmem + kColSf1, (j > 0 || kk > 0) ? 1u : 0u);
          }
        }
        tc_commit(&s.bar_pv_done);
        tc_commit(&s.bar_kv_empty[st]);
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int j = 0; ok && j < n_kv; ++j) {
        if (j + 1 < n_kv) ok = issue_s(j + 1);
        if (ok) ok = issue_pv(j);
      }
      // every MMA / copy issued above must complete before TMEM is released
      tc_commit(&s.bar_drain);
      drain_wait(&s.bar_drain, 0);
    }
  } else if (warp >= 4) {
    // ============================ softmax warpgroup ============================
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;                // row inside the tile == TMEM lane
    const int qrow = qt * kBM + r;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const float c = p.scale_log2;
    float m = -INFINITY;      // running max of the raw scores S
    float l = 0.f;            // running row sum
    bool ok = true;
    const bool dbg = p.dbg_codes != nullptr && bh_q == p.dbg_bh && qrow >= p.dbg_r0 && qrow < p.dbg_r1;
    uint8_t* p_row = s.p + r * (kBN / 2);
    const uint32_t swz = (static_cast<uint32_t>(r) >> 1) & 3u;

    for (int j = 0; j < n_kv; ++j) {
      const int sb = j & 1;
      ok = mbar_wait(&s.bar_s_full[sb], (j >> 1) & 1, abort_flag, p.status, kStatusTimeoutS | 8 | sb);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      float sv[kBN];
      {
        uint32_t raw[32];
#pragma unroll
        for (int cc = 0; cc < kBN / 32; ++cc) {
          tmem_ld32(tmem + lane_addr + (sb ? kColS1 : kColS0) + cc * 32, raw);
          tc_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) sv[cc * 32 + i] = __uint_as_float(raw[i]);
        }
      }
      tc_fence_before();
      mbar_arrive(&s.bar_s_empty[sb]);

      // masking: keys beyond N, and keys after the query row when causal
      const int key0 = j * kBN;
      if (key0 + kBN > p.N || (p.causal && key0 + kBN - 1 > qt * kBM)) {
#pragma unroll
        for (int i = 0; i < kBN; ++i) {
          const int key = key0 + i;
          if (key >= p.N || (p.causal && key > qrow)) sv[i] = -INFINITY;
        }
      }
      float bmax[kBN / 32];
#pragma unroll
      for (int bb = 0; bb < kBN / 32; ++bb) {
        float mx = sv[bb * 32];
#pragma unroll
        for (int i = 1; i < 32; ++i) mx = fmaxf(mx, sv[bb * 32 + i]);
        bmax[bb] = mx;
      }
      float tmax = bmax[0];
#pragma unroll
      for (int bb = 1; bb < kBN / 32; ++bb) tmax = fmaxf(tmax, bmax[bb]);
      const float m_new = fmaxf(m, tmax);
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      const float alpha = (m == -INFINITY) ? 0.f : ex2_approx((m - m_use) * c);

      uint32_t words[kBN / 8];          // 16 words = 64 bytes of codes for this row
      uint32_t sbytes = 0;
      float tile_sum = 0.f;
#pragma unroll
      for (int bb = 0; bb < kBN / 32; ++bb) {
        const float amax = ex2_approx((bmax[bb] - m_use) * c);     // 0 for an all-masked block
        const uint32_t byte = e8m0_scale_byte(amax, p.mode);
        sbytes |= byte << (8 * bb);
        const float neg_e = static_cast<float>(127 - static_cast<int>(byte));
        float y[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) y[i] = ex2_approx_ftz(fmaf(sv[bb * 32 + i] - m_use, c, neg_e));
#pragma unroll
        for (int w = 0; w < 4; ++w) words[bb * 4 + w] = cvt_e2m1x8(y + 8 * w);
        if (!p.pnq) {   // conventional row sum of the unquantized exponentials
          float bsum = 0.f;
#pragma unroll
          for (int i = 0; i < 32; ++i) bsum += y[i];
          tile_sum = fmaf(bsum, pow2_from_byte(byte), tile_sum);
        }
      }
      l = fmaf(alpha, l, tile_sum);      // (with PNQ the row sum accumulates in TMEM instead)

      // P~ buffer and O are free once the previous P~V product has completed
      if (j > 0) {
        ok = mbar_wait(&s.bar_pv_done, (j - 1) & 1, abort_flag, p.status, kStatusTimeoutPV);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
      }
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        const uint4 v4 = make_uint4(words[ch * 4], words[ch * 4 + 1], words[ch * 4 + 2], words[ch * 4 + 3]);
        *reinterpret_cast<uint4*>(p_row + ((ch ^ swz) << 4)) = v4;
      }
      *reinterpret_cast<uint32_t*>(s.psf + ((r & 31) * 16 + (r >> 5) * 4)) = sbytes;
      if (dbg) {
        uint4* dc = reinterpret_cast<uint4*>(p.dbg_codes + static_cast<size_t>(qrow - p.dbg_r0) * (p.Npad / 2) +
                                             j * (kBN / 2));
#pragma unroll
        for (int ch = 0; ch < 4; ++ch)
          dc[ch] = make_uint4(words[ch * 4], words[ch * 4 + 1], words[ch * 4 + 2], words[ch * 4 + 3]);
        *reinterpret_cast<uint32_t*>(p.dbg_scales + static_cast<size_t>(qrow - p.dbg_r0) * (p.Npad / 32) +
                                     j * 4) = sbytes;
      }
      fence_proxy_async_smem();

      // history rescale of O (only when some row of this warp saw its max move)
      if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t raw[32];
          tmem_ld32(tmem + lane_addr + kColO + cc * 32, raw);
          tc_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) raw[i] = __float_as_uint(__uint_as_float(raw[i]) * alpha);
          tmem_st32(tmem + lane_addr + kColO + cc * 32, raw);
        }
        if (p.pnq) {
          const uint32_t lv = tmem_ld1(tmem + lane_addr + kColL);
          tc_wait_ld();
          tmem_st1(tmem + lane_addr + kColL, __float_as_uint(__uint_as_float(lv) * alpha));
        }
        tc_wait_st();
      }
      tc_fence_before();
      mbar_arrive(&s.bar_p_full);
      m = m_new;
    }

    // ---- epilogue: out = O / l
    if (ok) {
      ok = mbar_wait(&s.bar_pv_done, (n_kv - 1) & 1, abort_flag, p.status, kStatusTimeoutPV | 1);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc_fence_after();
      if (p.pnq) {
        l = __uint_as_float(tmem_ld1(tmem + lane_addr + kColL));
        tc_wait_ld();
      }
      const float inv_l = 1.f / l;
      const bool store = qrow < p.N;
      const size_t orow = (static_cast<size_t>(bh_q) * p.N + (store ? qrow : 0)) * D;
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t raw[32];
        tmem_ld32(tmem + lane_addr + kColO + cc * 32, raw);
        tc_wait_ld();
        if (store) {
          if (p.out_bf16) {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + orow + cc * 32);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint32_t wv[4];
#pragma unroll
              for (int t = 0; t < 4; ++t) {
                const __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(raw[v * 8 + 2 * t]) * inv_l,
                                                                __uint_as_float(raw[v * 8 + 2 * t + 1]) * inv_l);
                wv[t] = *reinterpret_cast<const uint32_t*>(&h2);
              }
              dst[v] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
            }
          } else {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + orow + cc * 32);
#pragma unroll
            for (int v = 0; v < 8; ++v)
              dst[v] = make_float4(__uint_as_float(raw[4 * v]) * inv_l, __uint_as_float(raw[4 * v + 1]) * inv_l,
                                   __uint_as_float(raw[4 * v + 2]) * inv_l,
                                   __uint_as_float(raw[4 * v + 3]) * inv_l);
          }
        }
      }
    }
    tc_fence_before();
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D>
static cudaError_t launch_d(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                            const AttnParams& p, cudaStream_t stream) {
  const size_t smem = smem_bytes<D>();
  cudaError_t e = cudaFuncSetAttribute(mxattn_fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const unsigned grid = static_cast<unsigned>(p.B) * p.Hq * (p.Npad / kBM);
  mxattn_fwd_kernel<D><<<grid, kThreads, smem, stream>>>(tmQ, tmK, tmV, p);
  return cudaGetLastError();
}

cudaError_t launch_attention(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                             const AttnParams& p, int d, cudaStream_t stream) {
  if (d == 128) return launch_d<128>(tmQ, tmK, tmV, p, stream);
  if (d == 64) return launch_d<64>(tmQ, tmK, tmV, p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace mxattn

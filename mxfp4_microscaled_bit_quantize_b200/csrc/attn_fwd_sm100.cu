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
// One CTA owns one 128-query tile of one (batch, query head) and visits keys in tiles of
// kKvTile = 64 in increasing order (P~ codes depend on the running max in force, so tile width
// and order are part of the definition; the oracle takes the same width). Two CTAs share an SM:
// each allocates half of TMEM and their softmax phases drift apart, so one CTA's exponentials
// overlap the other's serial work (max, scale selection, stores, rescale).
// Warp roles (192 threads):
//   warp 0     TMA producer: Q tile once, then K / V^T tiles and their scale atoms into an
//              NSTAGE-deep shared-memory ring (mbarrier complete_tx).
//   warp 1     TMEM owner and MMA issuer (one thread): copies scale atoms to TMEM with
//              tcgen05.cp, issues S = QK^T, O += P~ V^T and (PNQ) L += P~ 1.
//   warps 2-5  softmax warpgroup, one thread per query row (TMEM lane = row): reads S with
//              tcgen05.ld (S is single-buffered: the MMA for the next tile starts as soon as the
//              row is in registers), updates the running max, computes P~ / 2^e per 32-key block,
//              quantizes it in registers, writes codes (32B-swizzled, the MMA operand layout)
//              and scale bytes to shared memory, rescales O and L in TMEM when the max moves,
//              and finally normalises and stores the output.
// TMEM (256 columns per CTA): S [0,64) O [64,64+d) L [192,208) scale atoms 208..243.
// The kernel is templated on the format: MXFP4 (the method) or, for comparison, NVFP4 (blocks of
// 16 with E4M3 scales for Q, K, V and P~; kind::mxf4nvf4 products, the non-power-of-two P~ scale
// folded into the exponent bias as -log2 s).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "mxattn_internal.h"
#include "sm100_ptx.cuh"

namespace mxattn {

constexpr int kBM = 128;          // query rows per CTA
constexpr int kBN = kKvTile;      // keys per KV tile (64)
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColS = 0, kColO = 64, kColL = 192;
// Q and K scale atoms: one per 64 (NVFP4) or 128 (MXFP4) contraction elements, 4 columns each.
constexpr uint32_t kColSfQ = 208, kColSfK = 216, kColSf1 = 224;
// P~ scale atoms alternate between two column sets by tile parity, V scale atoms (one per pair of
// 64-key tiles) by pair parity: tcgen05.cp into columns an earlier MMA still reads is not ordered
// behind that MMA, and the product of tile j may still run when the scales of tile j+1 are
// copied. The set written for tile j+1 was last read by a product no later than that of tile
// j-1, which the softmax has seen complete before it hands over tile j+1.
// NVFP4 gives every 64-key tile its own V atom, which then alternates by tile parity.
constexpr uint32_t kColSfV = 228, kColSfP = 236;   // + 4 * set
constexpr int kOnesRows = 16;     // N of the row-sum MMA: row 0 all ones, rows 1..15 zero
constexpr int kPRowBytes = kBN / 2;                  // 32 bytes of codes per P~ row
constexpr size_t kMinSmem = 80 * 1024;               // at most two CTAs per SM (TMEM halves)

static_assert(kBN == 64, "the 32B-swizzled P~ / V^T layouts below assume 64-key tiles");

template <int D>
struct Cfg {
  static constexpr int kStages = 8;
  static constexpr int kQRowBytes = D / 2;                 // packed E2M1 per Q/K row
  static constexpr int kQTileBytes = kBM * kQRowBytes;
  static constexpr int kKTileBytes = kBN * kQRowBytes;
  static constexpr int kVTileBytes = D * kPRowBytes;       // V^T: D rows of 64 keys
  static constexpr uint32_t kQKLayout = (D == 128) ? kLayoutSw64 : kLayoutSw32;
  static constexpr uint32_t kQKSbo = 8 * kQRowBytes;       // 8-row swizzle atom
};

template <int D>
struct __align__(1024) Smem {
  uint8_t q[Cfg<D>::kQTileBytes];
  uint8_t k[Cfg<D>::kStages][Cfg<D>::kKTileBytes];
  uint8_t v[Cfg<D>::kStages][Cfg<D>::kVTileBytes];
  uint8_t p[2][kBM * kPRowBytes];         // P~ codes, double-buffered by tile parity
  uint8_t ones[kOnesRows * kPRowBytes];
  uint8_t qsf[1024];                      // MXFP4: one atom; NVFP4: D / 64 atoms
  uint8_t ksf[Cfg<D>::kStages][1024];
  uint8_t vsf[Cfg<D>::kStages][512];
  uint8_t psf[2][512];
  uint8_t onesf[512];
  uint64_t bar_q;
  uint64_t bar_kv_full[Cfg<D>::kStages];
  uint64_t bar_kv_empty[Cfg<D>::kStages];
  uint64_t bar_s_full;
  uint64_t bar_s_empty;
  // P~ buffer b written by all 128 rows (tiles of parity b). One barrier per buffer: a fast
  // softmax warp may arrive for tile j+1 before a slow one has arrived for tile j.
  uint64_t bar_p_full[2];
  uint64_t bar_pv_done[2];                 // completions of PV of even / odd tiles
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

// max over 32 consecutive values with three-input max instructions
__device__ __forceinline__ float block_max32(const float* v) {
  float a0 = fmax3(v[0], v[1], v[2]);
  float a1 = fmax3(v[3], v[4], v[5]);
  float a2 = fmax3(v[6], v[7], v[8]);
  float a3 = fmax3(v[9], v[10], v[11]);
#pragma unroll
  for (int i = 12; i < 28; i += 8) {          // elements 12..27
    a0 = fmax3(a0, v[i], v[i + 1]);
    a1 = fmax3(a1, v[i + 2], v[i + 3]);
    a2 = fmax3(a2, v[i + 4], v[i + 5]);
    a3 = fmax3(a3, v[i + 6], v[i + 7]);
  }
  a0 = fmax3(a0, v[28], v[29]);                // elements 28..31
  a1 = fmax3(a1, v[30], v[31]);
  return fmaxf(fmax3(a0, a1, a2), a3);
}

// max over 16 consecutive values
__device__ __forceinline__ float block_max16(const float* v) {
  const float a0 = fmax3(v[0], v[1], v[2]), a1 = fmax3(v[3], v[4], v[5]), a2 = fmax3(v[6], v[7], v[8]);
  const float a3 = fmax3(v[9], v[10], v[11]), a4 = fmax3(v[12], v[13], v[14]);
  return fmaxf(fmax3(a0, a1, a2), fmax3(a3, a4, v[15]));
}

__device__ __forceinline__ float lg2_approx(float x) {
  float y;
  asm("lg2.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// NV = false: MXFP4 (blocks of 32, UE8M0, OCP or UOS exponent). NV = true: the NVFP4 comparison
// format for Q, K, V and P~ (blocks of 16, E4M3 scale = RNE(amax / 6)).
template <int D, bool PNQ, bool DBG, bool NV>
__global__ void __launch_bounds__(kThreads, 2)
    mxattn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using C = Cfg<D>;
  constexpr int NS = C::kStages;
  constexpr int kQKAtoms = NV ? D / 64 : 1;            // scale atoms per 128 Q or K rows
  constexpr uint32_t kQKSfBytes = kQKAtoms * 512;
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
  const int n_kv = p.causal ? min(2 * qt + 2, n_kv_all) : n_kv_all;

  if (threadIdx.x == 0) {
    mbar_init(&s.bar_q, 1);
    for (int i = 0; i < NS; ++i) {
      mbar_init(&s.bar_kv_full[i], 1);
      mbar_init(&s.bar_kv_empty[i], 1);
    }
    mbar_init(&s.bar_s_full, 1);
    mbar_init(&s.bar_s_empty, kBM);
    mbar_init(&s.bar_p_full[0], kBM);
    mbar_init(&s.bar_p_full[1], kBM);
    mbar_init(&s.bar_pv_done[0], 1);
    mbar_init(&s.bar_pv_done[1], 1);
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
    // The whole warp runs the loop (warp-uniform operands); one elected lane issues the copies.
    const bool leader = elect_one_sync();
    if (leader) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      mbar_arrive_expect_tx(&s.bar_q, C::kQTileBytes + kQKSfBytes);
      tma_load_2d(s.q, &tmQ, &s.bar_q, 0, bh_q * p.rows_per_head + qt * kBM);
      bulk_load(s.qsf, p.qsf + (static_cast<size_t>(bh_q) * n_qt + qt) * kQKSfBytes, kQKSfBytes, &s.bar_q);
    }
    __syncwarp();
    int issued = 0;
    for (int j = 0; j < n_kv; ++j) {
      const int st = j % NS;
      if (j >= NS) {
        bool ok = mbar_wait(&s.bar_kv_empty[st], ((j / NS) & 1) ^ 1, abort_flag, p.status,
                            kStatusTimeoutEmpty | st);
        if (!__all_sync(0xffffffffu, ok)) break;
      }
      if (leader) {
        // K scale atoms cover 128 keys: tiles 2t and 2t+1 share them, loaded with the even tile;
        // V atoms likewise for MXFP4, one per 64-key tile for NVFP4
        const bool atoms = (j & 1) == 0;
        const bool v_atom = NV || atoms;
        mbar_arrive_expect_tx(&s.bar_kv_full[st], C::kKTileBytes + C::kVTileBytes + (atoms ? kQKSfBytes : 0) +
                                                      (v_atom ? 512 : 0));
        tma_load_2d(s.k[st], &tmK, &s.bar_kv_full[st], 0, bh_kv * p.rows_per_head + j * kBN);
        tma_load_2d(s.v[st], &tmV, &s.bar_kv_full[st], j * kPRowBytes, bh_kv * D);
        if (atoms)
          bulk_load(s.ksf[st], p.ksf + (static_cast<size_t>(bh_kv) * n_qt + (j >> 1)) * kQKSfBytes, kQKSfBytes,
                    &s.bar_kv_full[st]);
        if (v_atom) {
          const size_t v_at = NV ? static_cast<size_t>(bh_kv) * (p.Npad / kBN) + j
                                 : static_cast<size_t>(bh_kv) * n_qt + (j >> 1);
          bulk_load(s.vsf[st], p.vsf + v_at * 512, 512, &s.bar_kv_full[st]);
        }
      }
      __syncwarp();
      issued = j + 1;
    }
    if (*abort_flag && leader) {
      // let every copy this warp started land before the CTA can exit
      drain_wait(&s.bar_q, 0);
      for (int j = (issued > NS ? issued - NS : 0); j < issued; ++j)
        drain_wait(&s.bar_kv_full[j % NS], (j / NS) & 1);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ============================ MMA issuer ============================
    // The whole warp runs the loop (warp-uniform descriptors); one elected lane issues every
    // tcgen05 operation and commit, so completion tracking stays with that thread.
    const uint64_t sf_desc_base = smem_desc(0, 0, 128, kLayoutNone);
    auto sf_desc = [&](const void* ptr) { return sf_desc_base | ((smem_u32(ptr) >> 4) & 0x3FFFu); };
    if (PNQ) {
      // ones operand (row 0 = code 1.0 for every key, rows 1..15 = 0) with unit scales
      uint32_t* ow = reinterpret_cast<uint32_t*>(s.ones);
      for (int i = lane; i < kOnesRows * kPRowBytes / 4; i += 32) ow[i] = (i < kPRowBytes / 4) ? 0x22222222u : 0u;
      uint32_t* sw = reinterpret_cast<uint32_t*>(s.onesf);
      for (int i = lane; i < 512 / 4; i += 32) sw[i] = NV ? 0x38383838u : 0x7F7F7F7Fu;   // E4M3 / E8M0 1.0
      fence_proxy_async_smem();
    }
    __syncwarp();
    const bool leader = elect_one_sync();
    bool ok = __all_sync(0xffffffffu, mbar_wait(&s.bar_q, 0, abort_flag, p.status, kStatusTimeoutQ));
    if (ok) {
      tc_fence_after();
      if (leader) {
#pragma unroll
        for (int a = 0; a < kQKAtoms; ++a) tc_cp_sf(tmem + kColSfQ + 4 * a, sf_desc(s.qsf + a * 512));
        if (PNQ) tc_cp_sf(tmem + kColSf1, sf_desc(s.onesf));
      }
      __syncwarp();
    }
    auto issue_s = [&](int j) -> bool {
      const int st = j % NS;
      if (!__all_sync(0xffffffffu, mbar_wait(&s.bar_kv_full[st], (j / NS) & 1, abort_flag, p.status,
                                             kStatusTimeoutKV | st)))
        return false;
      // S is single-buffered: the previous tile must be in the softmax registers
      if (j >= 1 && !__all_sync(0xffffffffu, mbar_wait(&s.bar_s_empty, (j - 1) & 1, abort_flag, p.status,
                                                       kStatusTimeoutS)))
        return false;
      tc_fence_after();
      const uint32_t qa = smem_u32(s.q), ka = smem_u32(s.k[st]);
      // keys of an odd tile are rows 64..127 of the scale atom: TMEM columns 2, 3 of it
      const uint32_t sfk = tmem + kColSfK + 2 * (j & 1);
      if (leader) {
        // the even tile brings the K atoms of the pair; S of the previous pair has completed
        if ((j & 1) == 0) {
#pragma unroll
          for (int a = 0; a < kQKAtoms; ++a) tc_cp_sf(tmem + kColSfK + 4 * a, sf_desc(s.ksf[st] + a * 512));
        }
#pragma unroll
        for (int kk = 0; kk < D / 64; ++kk) {
          const uint64_t ad = smem_desc(qa + kk * 32, 0, C::kQKSbo, C::kQKLayout);
          const uint64_t bd = smem_desc(ka + kk * 32, 0, C::kQKSbo, C::kQKLayout);
          if constexpr (NV)   // one atom (four 16-element blocks) per K = 64 step
            tc_mma_nvf4(tmem + kColS, ad, bd, idesc_nvf4(kBN), tmem + kColSfQ + 4 * kk, sfk + 4 * kk, kk > 0);
          else
            tc_mma_mxf4(tmem + kColS, ad, bd, idesc_mxf4(kBN, 2 * kk, 2 * kk), tmem + kColSfQ, sfk, kk > 0);
        }
        tc_commit(&s.bar_s_full);
      }
      __syncwarp();
      return true;
    };
    auto issue_pv = [&](int j) -> bool {
      const int st = j % NS;
      if (!__all_sync(0xffffffffu, mbar_wait(&s.bar_p_full[j & 1], (j >> 1) & 1, abort_flag, p.status, kStatusTimeoutP)))
        return false;
      tc_fence_after();
      const uint32_t pa = smem_u32(s.p[j & 1]), va = smem_u32(s.v[st]);
      const uint64_t ad = smem_desc(pa, 0, 8 * kPRowBytes, kLayoutSw32);
      const uint64_t bd = smem_desc(va, 0, 8 * kPRowBytes, kLayoutSw32);
      if (leader) {
        const uint32_t sfp = tmem + kColSfP + 4 * (j & 1);
        const uint32_t sfv = tmem + kColSfV + 4 * (NV ? (j & 1) : ((j >> 1) & 1));
        tc_cp_sf(sfp, sf_desc(s.psf[j & 1]));
        if (NV || (j & 1) == 0) tc_cp_sf(sfv, sf_desc(s.vsf[st]));   // MXFP4: the V atom of the tile pair
        if constexpr (NV) {
          tc_mma_nvf4(tmem + kColO, ad, bd, idesc_nvf4(D), sfp, sfv, j > 0 ? 1u : 0u);
          if (PNQ) {
            const uint64_t od = smem_desc(smem_u32(s.ones), 0, 8 * kPRowBytes, kLayoutSw32);
            tc_mma_nvf4(tmem + kColL, ad, od, idesc_nvf4(kOnesRows), sfp, tmem + kColSf1, j > 0 ? 1u : 0u);
          }
        } else {
          // this tile's 64 keys are blocks 0,1 (even tile) or 2,3 (odd tile) of the V scale atom
          tc_mma_mxf4(tmem + kColO, ad, bd, idesc_mxf4(D, 0, 2 * (j & 1)), sfp, sfv, j > 0 ? 1u : 0u);
          if (PNQ) {
            const uint64_t od = smem_desc(smem_u32(s.ones), 0, 8 * kPRowBytes, kLayoutSw32);
            tc_mma_mxf4(tmem + kColL, ad, od, idesc_mxf4(kOnesRows, 0, 0), sfp, tmem + kColSf1,
                        j > 0 ? 1u : 0u);
          }
        }
        tc_commit(&s.bar_pv_done[j & 1]);
        tc_commit(&s.bar_kv_empty[st]);
      }
      __syncwarp();
      return true;
    };
    if (ok) ok = issue_s(0);
    for (int j = 0; ok && j < n_kv; ++j) {
      if (j + 1 < n_kv) ok = issue_s(j + 1);
      if (ok) ok = issue_pv(j);
    }
    // every MMA / copy issued above must complete before TMEM is released
    if (leader) {
      tc_commit(&s.bar_drain);
      drain_wait(&s.bar_drain, 0);
    }
    __syncwarp();
  } else {
    // ============================ softmax warpgroup ============================
    const int quarter = warp & 3;                     // TMEM lane quarter this warp may access
    const int r = quarter * 32 + lane;                // row inside the tile == TMEM lane
    const int qrow = qt * kBM + r;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const float c = p.scale_log2;
    float m = -INFINITY;      // running max of the raw scores S
    float l = 0.f;            // running row sum (pnq = 0)
    bool ok = true;
    const bool dbg = DBG && bh_q == p.dbg_bh && qrow >= p.dbg_r0 && qrow < p.dbg_r1;
    const uint32_t p_row_off = r * kPRowBytes;
    const uint32_t psf_off = (r & 31) * 16 + (r >> 5) * 4;
    const uint32_t swz = (static_cast<uint32_t>(r) >> 2) & 1u;   // 32-byte swizzle of this row

    for (int j = 0; j < n_kv; ++j) {
      ok = mbar_wait(&s.bar_s_full, j & 1, abort_flag, p.status, kStatusTimeoutS | 8);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      float sv[kBN];
      {
        uint32_t raw0[32], raw1[32];
        tmem_ld32(tmem + lane_addr + kColS, raw0);
        tmem_ld32(tmem + lane_addr + kColS + 32, raw1);
        tc_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          sv[i] = __uint_as_float(raw0[i]);
          sv[32 + i] = __uint_as_float(raw1[i]);
        }
      }
      tc_fence_before();
      mbar_arrive(&s.bar_s_empty);

      // masking: keys beyond N, and keys after the query row when causal
      const int key0 = j * kBN;
      if (key0 + kBN > p.N || (p.causal && key0 + kBN - 1 > qt * kBM)) {
#pragma unroll
        for (int i = 0; i < kBN; ++i) {
          const int key = key0 + i;
          if (key >= p.N || (p.causal && key > qrow)) sv[i] = -INFINITY;
        }
      }
      // per block (32 keys for MXFP4, 16 for NVFP4): amax from the exact difference (1 for the
      // block that holds the max), the block's scale byte, and the exponent bias nb of
      // y = P~ / s = 2^(S c - m c - log2 s): one FFMA + one ex2 per element
      constexpr int kPB = NV ? 16 : 32;          // keys per P~ scale block
      constexpr int kNPB = kBN / kPB;
      float bmax[kNPB];
#pragma unroll
      for (int bb = 0; bb < kNPB; ++bb) bmax[bb] = NV ? block_max16(sv + bb * kPB) : block_max32(sv + bb * kPB);
      float tmax = bmax[0];
#pragma unroll
      for (int bb = 1; bb < kNPB; ++bb) tmax = fmaxf(tmax, bmax[bb]);
      const float m_new = fmaxf(m, tmax);
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      const float alpha = (m == -INFINITY) ? 0.f : ex2_approx((m - m_use) * c);

      uint32_t sbytes = 0;
      float nb[kNPB], bscale[kNPB];
#pragma unroll
      for (int bb = 0; bb < kNPB; ++bb) {
        const float amax = ex2_approx((bmax[bb] - m_use) * c);     // 0 for an all-masked block
        uint32_t byte;
        if constexpr (NV) {
          // s = E4M3(amax / 6) with both quotients correctly rounded. s = 0 (amax <= 6 * 2^-10):
          // y = P~ itself (every value below the 0.25 rounding threshold, so the codes are 0 as
          // the format wants) and the unquantized row sum still counts the block with weight 1
          byte = e4m3_byte(__fdiv_rn(amax, 6.0f));
          const float sb = e4m3_value(byte);
          bscale[bb] = sb > 0.f ? sb : 1.f;
          nb[bb] = sb > 0.f ? fmaf(-m_use, c, -lg2_approx(sb)) : -m_use * c;
        } else {
          byte = e8m0_scale_byte(amax, p.mode);
          bscale[bb] = pow2_from_byte(byte);
          nb[bb] = fmaf(-m_use, c, static_cast<float>(127 - static_cast<int>(byte)));
        }
        sbytes |= byte << (8 * bb);
      }
      float y[kBN];
#pragma unroll
      for (int i = 0; i < kBN; ++i) y[i] = ex2_approx_ftz(fmaf(sv[i], c, nb[i / kPB]));
      uint32_t words[kBN / 8];          // 8 words = 32 bytes of codes for this row
#pragma unroll
      for (int w = 0; w < kBN / 8; ++w) words[w] = cvt_e2m1x8(y + 8 * w);
      if (!PNQ) {   // conventional row sum of the unquantized exponentials
        float tile_sum = 0.f;
#pragma unroll
        for (int bb = 0; bb < kNPB; ++bb) {
          float b0 = 0.f, b1 = 0.f;
#pragma unroll
          for (int i = 0; i < kPB; i += 2) {
            b0 += y[bb * kPB + i];
            b1 += y[bb * kPB + i + 1];
          }
          tile_sum = fmaf(b0 + b1, bscale[bb], tile_sum);
        }
        l = fmaf(alpha, l, tile_sum);
      }

      // P~ buffer j&1 is free once the product of tile j-2 (its last reader) has completed
      const int pb = j & 1;
      if (j >= 2) {
        ok = mbar_wait(&s.bar_pv_done[pb], ((j >> 1) - 1) & 1, abort_flag, p.status, kStatusTimeoutPV);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
      }
      uint8_t* p_row = s.p[pb] + p_row_off;
#pragma unroll
      for (int bb = 0; bb < kBN / 32; ++bb) {
        const uint4 v4 = make_uint4(words[bb * 4], words[bb * 4 + 1], words[bb * 4 + 2], words[bb * 4 + 3]);
        *reinterpret_cast<uint4*>(p_row + ((bb ^ swz) << 4)) = v4;
      }
      if constexpr (NV)
        *reinterpret_cast<uint32_t*>(s.psf[pb] + psf_off) = sbytes;            // 4 blocks of 16 keys
      else
        *reinterpret_cast<uint16_t*>(s.psf[pb] + psf_off) = static_cast<uint16_t>(sbytes);
      if (DBG && dbg) {
        uint4* dc = reinterpret_cast<uint4*>(p.dbg_codes + static_cast<size_t>(qrow - p.dbg_r0) * (p.Npad / 2) +
                                             j * kPRowBytes);
#pragma unroll
        for (int bb = 0; bb < kBN / 32; ++bb)
          dc[bb] = make_uint4(words[bb * 4], words[bb * 4 + 1], words[bb * 4 + 2], words[bb * 4 + 3]);
        if constexpr (NV)
          *reinterpret_cast<uint32_t*>(p.dbg_scales + static_cast<size_t>(qrow - p.dbg_r0) * (p.Npad / 16) + j * 4) =
              sbytes;
        else
          *reinterpret_cast<uint16_t*>(p.dbg_scales + static_cast<size_t>(qrow - p.dbg_r0) * (p.Npad / 32) + j * 2) =
              static_cast<uint16_t>(sbytes);
      }
      fence_proxy_async_smem();

      // history rescale of O and L (only when some row of this warp saw its max move); O may only
      // be touched once the product of tile j-1 has landed in it
      if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
        ok = mbar_wait(&s.bar_pv_done[pb ^ 1], ((j - 1) >> 1) & 1, abort_flag, p.status, kStatusTimeoutPV | 4);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
#pragma unroll 1
        for (int cc = 0; cc < D / 32; cc += 2) {   // 64 columns per round trip
          uint32_t raw0[32], raw1[32];
          const uint32_t col = tmem + lane_addr + kColO + cc * 32;
          tmem_ld32(col, raw0);
          tmem_ld32(col + 32, raw1);
          tc_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            raw0[i] = __float_as_uint(__uint_as_float(raw0[i]) * alpha);
            raw1[i] = __float_as_uint(__uint_as_float(raw1[i]) * alpha);
          }
          tmem_st32(col, raw0);
          tmem_st32(col + 32, raw1);
        }
        if (PNQ) {
          const uint32_t lv = tmem_ld1(tmem + lane_addr + kColL);
          tc_wait_ld();
          tmem_st1(tmem + lane_addr + kColL, __float_as_uint(__uint_as_float(lv) * alpha));
        }
        tc_wait_st();
      }
      tc_fence_before();
      mbar_arrive(&s.bar_p_full[pb]);
      m = m_new;
    }

    // ---- epilogue: out = O / l (PV products complete in order: the last one covers all)
    if (ok) {
      ok = mbar_wait(&s.bar_pv_done[(n_kv - 1) & 1], ((n_kv - 1) >> 1) & 1, abort_flag, p.status,
                     kStatusTimeoutPV | 1);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc_fence_after();
      if (PNQ) {
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

template <int D, bool PNQ, bool DBG, bool NV>
static cudaError_t launch_k(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                            const AttnParams& p, cudaStream_t stream) {
  const size_t smem = smem_bytes<D>();
  cudaError_t e = cudaFuncSetAttribute(mxattn_fwd_kernel<D, PNQ, DBG, NV>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const unsigned grid = static_cast<unsigned>(p.B) * p.Hq * (p.Npad / kBM);
  mxattn_fwd_kernel<D, PNQ, DBG, NV><<<grid, kThreads, smem, stream>>>(tmQ, tmK, tmV, p);
  return cudaGetLastError();
}

template <int D, bool NV>
static cudaError_t launch_f(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                            const AttnParams& p, cudaStream_t stream) {
  const bool dbg = p.dbg_codes != nullptr;
  if (p.pnq) return dbg ? launch_k<D, true, true, NV>(tmQ, tmK, tmV, p, stream)
                        : launch_k<D, true, false, NV>(tmQ, tmK, tmV, p, stream);
  return dbg ? launch_k<D, false, true, NV>(tmQ, tmK, tmV, p, stream)
             : launch_k<D, false, false, NV>(tmQ, tmK, tmV, p, stream);
}

template <int D>
static cudaError_t launch_d(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                            const AttnParams& p, cudaStream_t stream) {
  return p.mode == kModeNvfp4 ? launch_f<D, true>(tmQ, tmK, tmV, p, stream)
                              : launch_f<D, false>(tmQ, tmK, tmV, p, stream);
}

cudaError_t launch_attention(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                             const AttnParams& p, int d, cudaStream_t stream) {
  if (d == 128) return launch_d<128>(tmQ, tmK, tmV, p, stream);
  if (d == 64) return launch_d<64>(tmQ, tmK, tmV, p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace mxattn

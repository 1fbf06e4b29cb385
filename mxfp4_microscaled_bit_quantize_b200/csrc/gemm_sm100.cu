// Block-scaled MXFP4 GEMM for sm_100a: C[M, N] = dq(A)[M, K] dq(B)[N, K]^T with both operands
// in MXFP4 (E2M1 codes, one E8M0 scale per 32 elements along K), fp32 accumulation in TMEM.
//
// What it computes: the MX block format of the "Quantization Error" page (section "Where the
// error comes from": exact power-of-two scales, one rounding step per element) applied to both
// operands of a matrix product, the W4A4 setting the MXCode digest describes (MX-native operands
// fed to the tensor cores), without its VQ codebooks. Each 32-element block contributes
// 2^(ea + eb) * sum(ca * cb) exactly; the tensor core accumulates blocks in fp32.
//
// Persistent kernel: one CTA per SM walks 128 x 256 tiles of C in groups of kGroupM tile rows
// (so the A and B slices in flight at once stay in L2). Roles:
//   warp 0     TMA producer: K slices of 256 elements (128 bytes of codes per row) of A (128 rows)
//              and B (256 rows), 128-byte swizzle, into a 4-stage (NVFP4: 3) ring that runs across
//              tile boundaries, plus their scale atoms (512 bytes per 128 rows x 128 K elements).
//   warp 1     TMEM owner and MMA issuer: tcgen05.cp moves the scale atoms of a stage into that
//              stage's own TMEM columns (a copy is not ordered behind earlier MMAs that read the
//              same columns; a stage's columns are rewritten only after the ring has recycled the
//              stage, i.e. after its MMAs completed), then 4 x tcgen05.mma kind::mxf4.block_scale
//              (M = 128, N = 256, K = 64) per stage. A tile starts once the epilogue has drained
//              the previous tile's accumulator.
//   warps 2-5  epilogue, one accumulator row per thread. bf16: tcgen05.ld the whole row into
//              registers (packed bf16), release the accumulator, then stream the row out through a
//              128-byte-swizzled staging box in shared memory, one TMA store per 64 columns, while
//              the next tile's MMAs run. fp32: direct row stores, then release.
// TMEM: accumulator columns [0, 256), scale columns from 256 (12 per scale atom of a stage).
// Templated on the format: MXFP4 (blocks of 32, UE8M0, kind::mxf4) or NVFP4 (blocks of 16, UE4M3,
// kind::mxf4nvf4: twice the scale atoms per K, so a 3-stage ring).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "mxattn_internal.h"
#include "sm100_ptx.cuh"

namespace mxattn {
namespace {

constexpr int kGm = 128;              // rows of A per tile
constexpr int kGn = 256;              // rows of B (columns of C) per tile
constexpr int kGk = 256;              // K elements per stage
constexpr int kGkBytes = kGk / 2;     // 128 bytes of codes per row per stage
constexpr int kGroupM = 8;            // tile rows per raster group
constexpr int kGThreads = 192;
constexpr uint32_t kGTmemCols = 512;
constexpr uint32_t kGColAcc = 0;
constexpr uint32_t kGColSf = 256;     // + stage * kKg * 12 + kgroup * 12: SFA 4 columns, SFB 8 columns
constexpr uint32_t kLayoutSw128 = 2;  // shared-memory descriptor layout code of the 128-byte swizzle
constexpr int kCBoxCols = 64;         // bf16 columns per TMA store box (128 bytes)

// Per format: MXFP4 (blocks of 32, UE8M0): a scale atom covers 128 K elements, two per stage, two
// K = 64 MMAs per atom. NVFP4 (blocks of 16, UE4M3): an atom covers 64 K elements, four per stage,
// one MMA per atom; its larger scale footprint leaves room for one stage less.
template <bool NV>
struct GemmFmt {
  static constexpr int kStages = NV ? 3 : 4;
  static constexpr int kKg = NV ? 4 : 2;          // scale atoms (K groups) per stage
  static constexpr int kMmaPerKg = NV ? 1 : 2;
};

template <bool NV>
struct __align__(1024) GemmSmem {
  static constexpr int S = GemmFmt<NV>::kStages, G = GemmFmt<NV>::kKg;
  uint8_t a[S][kGm * kGkBytes];            // 16 KiB per stage
  uint8_t b[S][kGn * kGkBytes];            // 32 KiB per stage
  uint8_t c[kGm * 128];                    // bf16 staging box: 128 rows x 64 columns, 128B swizzle
  uint8_t sfa[S][G][512];                  // [kgroup] atom of the 128 A rows
  uint8_t sfb[S][2][G][512];               // [row tile][kgroup]
  uint64_t full[S];
  uint64_t empty[S];
  uint64_t acc_full;                       // MMA -> epilogue, once per tile
  uint64_t acc_empty;                      // epilogue (128 threads) -> MMA, once per tile
  uint64_t c_written;                      // epilogue threads (128) -> store thread, once per box
  uint64_t c_free;                         // store thread -> epilogue: staging box read by TMA
  uint32_t tmem_base;
  int abort_flag;
};

template <bool NV>
constexpr size_t gemm_smem_bytes() { return sizeof(GemmSmem<NV>) + 1024; }
static_assert(gemm_smem_bytes<false>() <= 232448 && gemm_smem_bytes<true>() <= 232448, "shared memory per CTA");

__device__ __forceinline__ void gemm_drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > 200ull * 1000ull * 1000ull) break;
  }
}

// Tile t of the grouped raster: kGroupM tile rows at a time, down the rows first.
__device__ __forceinline__ void tile_coords(int t, int tiles_m, int tiles_n, int& tm, int& tn) {
  const int per_group = kGroupM * tiles_n;
  const int g = t / per_group;
  const int first_m = g * kGroupM;
  const int gm = min(kGroupM, tiles_m - first_m);
  const int r = t - g * per_group;
  tm = first_m + r % gm;
  tn = r / gm;
}

template <bool NV>
__global__ void __launch_bounds__(kGThreads, 1)
    mxgemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                  const __grid_constant__ CUtensorMap tmC, const GemmParams p) {
  constexpr int kGStages = GemmFmt<NV>::kStages;
  constexpr int kKg = GemmFmt<NV>::kKg;
  constexpr uint32_t kSfBytes = 3u * kKg * 512u;   // A atoms + two row tiles of B atoms per stage
  extern __shared__ uint8_t smem_raw[];
  GemmSmem<NV>& s =
      *reinterpret_cast<GemmSmem<NV>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_k = p.k_stages;
  const int tiles_m = (p.M + kGm - 1) / kGm;
  const int tiles_n = (p.N + kGn - 1) / kGn;
  const int n_tiles = tiles_m * tiles_n;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kGStages; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    mbar_init(&s.acc_full, 1);
    mbar_init(&s.acc_empty, 128);
    mbar_init(&s.c_written, 128);
    mbar_init(&s.c_free, 1);
    s.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&s.tmem_base, kGTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  volatile int* abort_flag = &s.abort_flag;

  if (warp == 0) {
    // ============================ TMA producer ============================
    const bool leader = elect_one_sync();
    if (leader) {
      prefetch_tmap(&tmA);
      prefetch_tmap(&tmB);
    }
    int it = 0;    // k slices issued so far, across tiles
    bool ok = true;
    for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x) {
      int tm, tn;
      tile_coords(t, tiles_m, tiles_n, tm, tn);
      for (int kt = 0; kt < n_k; ++kt) {
        const int st = it % kGStages;
        if (it >= kGStages) {
          ok = __all_sync(0xffffffffu, mbar_wait(&s.empty[st], ((it / kGStages) & 1) ^ 1, abort_flag, p.status,
                                                 kStatusTimeoutEmpty | st));
          if (!ok) break;
        }
        if (leader) {
          mbar_arrive_expect_tx(&s.full[st], kGm * kGkBytes + kGn * kGkBytes + kSfBytes);
          tma_load_2d(s.a[st], &tmA, &s.full[st], kt * kGkBytes, tm * kGm);
          tma_load_2d(s.b[st], &tmB, &s.full[st], kt * kGkBytes, tn * kGn);
          // atoms [row tile][kgroup][512]: the kgroups of this stage are adjacent
          const size_t kg = static_cast<size_t>(kKg) * kt;
          bulk_load(s.sfa[st][0], p.sfa + (static_cast<size_t>(tm) * p.kgroups + kg) * 512, kKg * 512, &s.full[st]);
          for (int rt = 0; rt < 2; ++rt)
            bulk_load(s.sfb[st][rt][0], p.sfb + (static_cast<size_t>(2 * tn + rt) * p.kgroups + kg) * 512, kKg * 512,
                      &s.full[st]);
        }
        __syncwarp();
        ++it;
      }
    }
    if (*abort_flag && leader) {
      for (int k = (it > kGStages ? it - kGStages : 0); k < it; ++k)
        gemm_drain_wait(&s.full[k % kGStages], (k / kGStages) & 1);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ============================ MMA issuer ============================
    const bool leader = elect_one_sync();
    const uint64_t sf_desc_base = smem_desc(0, 0, 128, kLayoutNone);
    auto sf_desc = [&](const void* ptr) { return sf_desc_base | ((smem_u32(ptr) >> 4) & 0x3FFFu); };
    constexpr uint32_t idesc0 = NV ? idesc_nvf4(kGn) : idesc_mxf4(kGn, 0, 0);
    constexpr uint32_t idesc1 = idesc_mxf4(kGn, 2, 2);
    // per-stage descriptors, computed once: a K step inside the 128-byte swizzled rows only adds
    // (offset >> 4) to the start-address field (shared addresses stay below 2^18, no carry)
    uint64_t desc_a[kGStages], desc_b[kGStages], desc_sfa[kGStages][kKg], desc_sfb[kGStages][2][kKg];
#pragma unroll
    for (int st = 0; st < kGStages; ++st) {
      desc_a[st] = smem_desc(smem_u32(s.a[st]), 0, 8 * kGkBytes, kLayoutSw128);
      desc_b[st] = smem_desc(smem_u32(s.b[st]), 0, 8 * kGkBytes, kLayoutSw128);
#pragma unroll
      for (int g = 0; g < kKg; ++g) {
        desc_sfa[st][g] = sf_desc(s.sfa[st][g]);
        desc_sfb[st][0][g] = sf_desc(s.sfb[st][0][g]);
        desc_sfb[st][1][g] = sf_desc(s.sfb[st][1][g]);
      }
    }
    bool ok = true;
    int it = 0, i = 0;
    for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x, ++i) {
      if (i > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(&s.acc_empty, (i - 1) & 1, abort_flag, p.status,
                                               kStatusTimeoutS | 1));
        if (!ok) break;
        tc_fence_after();
      }
      for (int kt = 0; kt < n_k; ++kt, ++it) {
        const int st = it % kGStages;
        ok = __all_sync(0xffffffffu, mbar_wait(&s.full[st], (it / kGStages) & 1, abort_flag, p.status,
                                               kStatusTimeoutKV | st));
        if (!ok) break;
        tc_fence_after();
        if (leader) {
          uint64_t da = 0, db = 0, dsa[kKg], dsb[2][kKg];
#pragma unroll
          for (int g = 0; g < kKg; ++g) dsa[g] = dsb[0][g] = dsb[1][g] = 0;
#pragma unroll
          for (int q = 0; q < kGStages; ++q) {   // select this stage's descriptors without local memory
            if (q == st) {
              da = desc_a[q];
              db = desc_b[q];
#pragma unroll
              for (int g = 0; g < kKg; ++g) {
                dsa[g] = desc_sfa[q][g];
                dsb[0][g] = desc_sfb[q][0][g];
                dsb[1][g] = desc_sfb[q][1][g];
              }
            }
          }
#pragma unroll
          for (int g = 0; g < kKg; ++g) {
            const uint32_t sfa = tmem + kGColSf + (st * kKg + g) * 12, sfb = sfa + 4;
            tc_cp_sf(sfa, dsa[g]);
            tc_cp_sf(sfb, dsb[0][g]);
            tc_cp_sf(sfb + 4, dsb[1][g]);
#pragma unroll
            for (int kk = 0; kk < GemmFmt<NV>::kMmaPerKg; ++kk) {
              // K offset of this instruction inside the 128-byte rows: 64 K elements = 32 bytes
              const uint64_t off = static_cast<uint64_t>((g * 32 * GemmFmt<NV>::kMmaPerKg + kk * 32) >> 4);
              if constexpr (NV)
                tc_mma_nvf4(tmem + kGColAcc, da + off, db + off, idesc0, sfa, sfb, (kt | g) != 0 ? 1u : 0u);
              else
                tc_mma_mxf4(tmem + kGColAcc, da + off, db + off, kk ? idesc1 : idesc0, sfa, sfb,
                            (kt | g | kk) != 0 ? 1u : 0u);
            }
          }
          tc_commit(&s.empty[st]);   // the stage's smem and scale columns are free once these MMAs end
        }
        __syncwarp();
      }
      if (ok && leader) tc_commit(&s.acc_full);   // every MMA of the tile
      __syncwarp();
    }
    if (!ok && leader) {
      // let every MMA this thread issued finish before TMEM is released: a fresh commit tracks
      // all of them; its arrival lands on acc_full, which nobody waits on any more
      tc_commit(&s.acc_full);
      gemm_drain_wait(&s.acc_full, static_cast<uint32_t>(i & 1));
    }
    __syncwarp();
  } else {
    // ============================ epilogue ============================
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;                 // row inside the tile == TMEM lane
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const bool store_thread = threadIdx.x == 64;
    const uint32_t swz = static_cast<uint32_t>(r) & 7u;
    int i = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x, ++i) {
      int tm, tn;
      tile_coords(t, tiles_m, tiles_n, tm, tn);
      ok = __all_sync(0xffffffffu, mbar_wait(&s.acc_full, i & 1, abort_flag, p.status, kStatusTimeoutPV | 1));
      if (!ok) break;
      if (p.out_bf16) {
        tc_fence_after();
        uint32_t packed[kGn / 2];            // the row as bf16 pairs
#pragma unroll
        for (int cc = 0; cc < kGn / 32; ++cc) {
          uint32_t raw[32];
          tmem_ld32(tmem + lane_addr + kGColAcc + cc * 32, raw);
          tc_wait_ld();
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            const __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(raw[2 * u]), __uint_as_float(raw[2 * u + 1]));
            packed[cc * 16 + u] = *reinterpret_cast<const uint32_t*>(&h2);
          }
        }
        tc_fence_before();
        mbar_arrive(&s.acc_empty);           // the MMAs of the next tile may overwrite TMEM now
        uint8_t* row_base = s.c + r * 128;
#pragma unroll
        for (int b = 0; b < kGn / kCBoxCols; ++b) {
          const int seq = i * (kGn / kCBoxCols) + b;   // staging box uses so far
          if (seq > 0) {   // the previous store must have read the staging box
            ok = __all_sync(0xffffffffu, mbar_wait(&s.c_free, (seq - 1) & 1, abort_flag, p.status, kStatusTimeoutPV | 2));
            if (!ok) break;
          }
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint32_t* w = packed + b * 32 + j * 4;
            *reinterpret_cast<uint4*>(row_base + ((static_cast<uint32_t>(j) ^ swz) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
          }
          fence_proxy_async_smem();          // staging writes -> visible to the TMA store
          mbar_arrive(&s.c_written);
          if (store_thread) {
            if (mbar_wait(&s.c_written, seq & 1, abort_flag, p.status, kStatusTimeoutPV | 3)) {
              const int x = tn * kGn + b * kCBoxCols;
              if (x < p.N) tma_store_2d(&tmC, s.c, x, tm * kGm);
              bulk_commit_group();
              bulk_wait_group_read0();
              mbar_arrive(&s.c_free);
            }
          }
          __syncwarp();
        }
        if (!ok) break;
      } else {
        tc_fence_after();
        const int row = tm * kGm + r;
        const bool row_ok = row < p.M;
#pragma unroll 1
        for (int cc = 0; cc < kGn / 32; ++cc) {
          uint32_t raw[32];
          tmem_ld32(tmem + lane_addr + kGColAcc + cc * 32, raw);
          tc_wait_ld();
          const int col0 = tn * kGn + cc * 32;
          const size_t base = static_cast<size_t>(row) * p.N + col0;
          if (!row_ok || col0 >= p.N) {
            // nothing of this chunk is inside C
          } else if (col0 + 32 <= p.N) {   // N % 8 == 0: 16-byte aligned row chunks
            uint4* dst = reinterpret_cast<uint4*>(static_cast<float*>(p.c) + base);
#pragma unroll
            for (int v = 0; v < 8; ++v) dst[v] = make_uint4(raw[4 * v], raw[4 * v + 1], raw[4 * v + 2], raw[4 * v + 3]);
          } else {
#pragma unroll
            for (int u = 0; u < 32; ++u) {
              if (col0 + u >= p.N) break;
              static_cast<float*>(p.c)[base + u] = __uint_as_float(raw[u]);
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&s.acc_empty);
      }
    }
    if (store_thread) bulk_wait_group0();   // every TMA store of C has completed
    __syncwarp();
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kGTmemCols);
  }
}

template <bool NV>
cudaError_t launch_gemm_fmt(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmC,
                            const GemmParams& p, cudaStream_t stream) {
  constexpr size_t smem = gemm_smem_bytes<NV>();
  cudaError_t e = cudaFuncSetAttribute(mxgemm_kernel<NV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long tiles = static_cast<long>((p.M + kGm - 1) / kGm) * ((p.N + kGn - 1) / kGn);
  const unsigned grid = static_cast<unsigned>(tiles < sms ? tiles : sms);
  mxgemm_kernel<NV><<<grid, kGThreads, smem, stream>>>(tmA, tmB, tmC, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmC, const GemmParams& p,
                        cudaStream_t stream) {
  return p.nvfp4 ? launch_gemm_fmt<true>(tmA, tmB, tmC, p, stream) : launch_gemm_fmt<false>(tmA, tmB, tmC, p, stream);
}

}  // namespace mxattn

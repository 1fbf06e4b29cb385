// Block-scaled MXFP4 GEMM for sm_100a: C[M, N] = dq(A)[M, K] dq(B)[N, K]^T with both operands
// in MXFP4 (E2M1 codes, one E8M0 scale per 32 elements along K), fp32 accumulation in TMEM.
//
// What it computes: the MX block format of the "Quantization Error" page (section "Where the
// error comes from": exact power-of-two scales, one rounding step per element) applied to both
// operands of a matrix product, the W4A4 setting the MXCode digest describes (MX-native operands
// fed to the tensor cores), without its VQ codebooks. Each 32-element block contributes
// 2^(ea + eb) * sum(ca * cb) exactly; the tensor core accumulates blocks in fp32.
//
// One CTA computes one 128 x 256 tile of C:
//   warp 0     TMA producer: K slices of 256 elements (128 bytes of codes per row) of A (128 rows)
//              and B (256 rows), 128-byte swizzle, into a kStages-deep ring, plus their scale
//              atoms (512 bytes per 128 rows x 128 K elements) by bulk copy.
//   warp 1     TMEM owner and MMA issuer: tcgen05.cp moves the scale atoms of a stage into that
//              stage's own TMEM columns (a copy is not ordered behind earlier MMAs that read the
//              same columns; a stage's columns are rewritten only after the ring has recycled the
//              stage, i.e. after its MMAs completed), then 4 x tcgen05.mma kind::mxf4.block_scale
//              (M = 128, N = 256, K = 64) per stage.
//   warps 2-5  epilogue: tcgen05.ld of the accumulator (one row per thread) and stores of fp32 or
//              bf16 rows of C.
// TMEM: accumulator columns [0, 256), scale columns from 256 (kStages x 24).
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
constexpr int kGStages = 4;
constexpr int kGThreads = 192;
constexpr uint32_t kGTmemCols = 512;
constexpr uint32_t kGColAcc = 0;
constexpr uint32_t kGColSf = 256;     // + stage * 24 + kgroup * 12: SFA 4 columns, SFB 8 columns
constexpr uint32_t kLayoutSw128 = 2;  // shared-memory descriptor layout code of the 128-byte swizzle

struct __align__(1024) GemmSmem {
  uint8_t a[kGStages][kGm * kGkBytes];     // 16 KiB per stage
  uint8_t b[kGStages][kGn * kGkBytes];     // 32 KiB per stage
  uint8_t sfa[kGStages][2][512];           // [kgroup] atom of the 128 A rows
  uint8_t sfb[kGStages][2][2][512];        // [row tile][kgroup]
  uint64_t full[kGStages];
  uint64_t empty[kGStages];
  uint64_t acc_full;
  uint32_t tmem_base;
  int abort_flag;
};

constexpr size_t kGemmSmemBytes = sizeof(GemmSmem) + 1024;

__device__ __forceinline__ void gemm_drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > 200ull * 1000ull * 1000ull) break;
  }
}

__global__ void __launch_bounds__(kGThreads, 1)
    mxgemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                  const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  GemmSmem& s = *reinterpret_cast<GemmSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tile_n = blockIdx.x;
  const int tile_m = blockIdx.y;
  const int n_k = p.k_stages;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kGStages; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    mbar_init(&s.acc_full, 1);
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
    int issued = 0;
    for (int kt = 0; kt < n_k; ++kt) {
      const int st = kt % kGStages;
      if (kt >= kGStages) {
        const bool ok = mbar_wait(&s.empty[st], ((kt / kGStages) & 1) ^ 1, abort_flag, p.status,
                                  kStatusTimeoutEmpty | st);
        if (!__all_sync(0xffffffffu, ok)) break;
      }
      if (leader) {
        mbar_arrive_expect_tx(&s.full[st], kGm * kGkBytes + kGn * kGkBytes + 3 * 1024);
        tma_load_2d(s.a[st], &tmA, &s.full[st], kt * kGkBytes, tile_m * kGm);
        tma_load_2d(s.b[st], &tmB, &s.full[st], kt * kGkBytes, tile_n * kGn);
        // atoms [row tile][kgroup][512]: the two kgroups of this stage are adjacent
        const size_t kg = static_cast<size_t>(2 * kt);
        bulk_load(s.sfa[st][0], p.sfa + (static_cast<size_t>(tile_m) * p.kgroups + kg) * 512, 1024, &s.full[st]);
        for (int rt = 0; rt < 2; ++rt)
          bulk_load(s.sfb[st][rt][0], p.sfb + (static_cast<size_t>(2 * tile_n + rt) * p.kgroups + kg) * 512, 1024,
                    &s.full[st]);
      }
      __syncwarp();
      issued = kt + 1;
    }
    if (*abort_flag && leader) {
      for (int kt = (issued > kGStages ? issued - kGStages : 0); kt < issued; ++kt)
        gemm_drain_wait(&s.full[kt % kGStages], (kt / kGStages) & 1);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ============================ MMA issuer ============================
    const bool leader = elect_one_sync();
    const uint64_t sf_desc_base = smem_desc(0, 0, 128, kLayoutNone);
    auto sf_desc = [&](const void* ptr) { return sf_desc_base | ((smem_u32(ptr) >> 4) & 0x3FFFu); };
    constexpr uint32_t idesc0 = idesc_mxf4(kGn, 0, 0);
    constexpr uint32_t idesc1 = idesc_mxf4(kGn, 2, 2);
    bool ok = true;
    for (int kt = 0; kt < n_k; ++kt) {
      const int st = kt % kGStages;
      ok = __all_sync(0xffffffffu, mbar_wait(&s.full[st], (kt / kGStages) & 1, abort_flag, p.status,
                                             kStatusTimeoutKV | st));
      if (!ok) break;
      tc_fence_after();
      if (leader) {
        const uint32_t a0 = smem_u32(s.a[st]), b0 = smem_u32(s.b[st]);
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          const uint32_t sfa = tmem + kGColSf + st * 24 + g * 12, sfb = sfa + 4;
          tc_cp_sf(sfa, sf_desc(s.sfa[st][g]));
          tc_cp_sf(sfb, sf_desc(s.sfb[st][0][g]));
          tc_cp_sf(sfb + 4, sf_desc(s.sfb[st][1][g]));
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) {
            const uint32_t off = g * 64 + kk * 32;
            const uint64_t ad = smem_desc(a0 + off, 0, 8 * kGkBytes, kLayoutSw128);
            const uint64_t bd = smem_desc(b0 + off, 0, 8 * kGkBytes, kLayoutSw128);
            tc_mma_mxf4(tmem + kGColAcc, ad, bd, kk ? idesc1 : idesc0, sfa, sfb, (kt | g | kk) != 0 ? 1u : 0u);
          }
        }
        tc_commit(&s.empty[st]);   // the stage's smem and scale columns are free once these MMAs end
      }
      __syncwarp();
    }
    if (leader) {
      tc_commit(&s.acc_full);      // every MMA above, or on abort whatever was issued
    }
    __syncwarp();
    if (!ok && leader) gemm_drain_wait(&s.acc_full, 0);
  } else {
    // ============================ epilogue ============================
    const int quarter = warp & 3;
    const int row = tile_m * kGm + quarter * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    bool ok = mbar_wait(&s.acc_full, 0, abort_flag, p.status, kStatusTimeoutPV | 1);
    ok = __all_sync(0xffffffffu, ok) && !*abort_flag;
    if (ok) {
      tc_fence_after();
      const bool row_ok = row < p.M;
#pragma unroll 1
      for (int cc = 0; cc < kGn / 32; ++cc) {
        uint32_t raw[32];
        tmem_ld32(tmem + lane_addr + kGColAcc + cc * 32, raw);
        tc_wait_ld();
        const int col0 = tile_n * kGn + cc * 32;
        const size_t base = static_cast<size_t>(row) * p.N + col0;
        if (!row_ok || col0 >= p.N) {
          // nothing of this chunk is inside C
        } else if (col0 + 32 <= p.N) {   // N % 8 == 0: 16-byte aligned row chunks
          if (p.out_bf16) {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.c) + base);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint32_t w[4];
#pragma unroll
              for (int t = 0; t < 4; ++t) {
                const __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(raw[v * 8 + 2 * t]),
                                                                __uint_as_float(raw[v * 8 + 2 * t + 1]));
                w[t] = *reinterpret_cast<const uint32_t*>(&h2);
              }
              dst[v] = make_uint4(w[0], w[1], w[2], w[3]);
            }
          } else {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<float*>(p.c) + base);
#pragma unroll
            for (int v = 0; v < 8; ++v) dst[v] = make_uint4(raw[4 * v], raw[4 * v + 1], raw[4 * v + 2], raw[4 * v + 3]);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            if (col0 + i >= p.N) break;
            if (p.out_bf16)
              static_cast<__nv_bfloat16*>(p.c)[base + i] = __float2bfloat16_rn(__uint_as_float(raw[i]));
            else
              static_cast<float*>(p.c)[base + i] = __uint_as_float(raw[i]);
          }
        }
      }
    }
    tc_fence_before();
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kGTmemCols);
  }
}

}  // namespace

cudaError_t launch_gemm(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmParams& p, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(mxgemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kGemmSmemBytes));
  if (e != cudaSuccess) return e;
  dim3 grid(static_cast<unsigned>((p.N + kGn - 1) / kGn), static_cast<unsigned>((p.M + kGm - 1) / kGm));
  mxgemm_kernel<<<grid, kGThreads, kGemmSmemBytes, stream>>>(tmA, tmB, p);
  return cudaGetLastError();
}

}  // namespace mxattn

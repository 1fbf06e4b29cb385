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
// Work unit: one CTA (one per SM: it allocates all 512 TMEM columns) owns two consecutive
// 128-query tiles A and B of one (batch, query head) and visits keys in tiles of kKvTile = 128 in
// increasing order (P~ codes depend on the running max in force, so tile width and order are part
// of the definition; the oracle takes the same width). The two query tiles share every K / V^T
// tile in shared memory and take turns on ONE 128-column S buffer in TMEM: S(A, t), S(B, t),
// S(A, t+1), ... . Their softmax warps therefore run half a step apart, and on every SM
// sub-partition one tile's serial work (S load, maxima, scale selection, stores, rescale) overlaps
// the other tile's exponentials on the MUFU.
// Warp roles (control warpgroup 0, then the softmax warpgroups; the layout WS is chosen per
// launch, see Layout and launch_w):
//   warp 2     TMA producer: Q tiles A and B once, then K / V^T tiles and their scale atoms into
//              an NSTAGE-deep shared-memory ring (mbarrier complete_tx).
//   warp 1     TMEM owner and S issuer (one thread): copies the Q and K scale atoms and issues
//              S(A, t), S(B, t), S(A, t+1), ..., each once the previous user of the S buffer holds
//              its scores in registers.
//   warps 0, 3 P~V issuers of tiles A and B (one thread each): copy the P~ and V scale atoms to
//              TMEM and issue O_X += P~_X(t) V(t) and L_X += P~_X(t) 1 as soon as tile X's softmax
//              hands P~ over. The four control warps sit on the four SM sub-partitions, so that the
//              tcgen05 issue work is spread next to all eight softmax warps, which set the pace.
//   WS = 4     warps 4-7 softmax of tile A, warps 8-11 of tile B (384 threads): one thread per
//              query row (TMEM lane = row). Per key tile a thread reads its 128 scores with
//              tcgen05.ld, releases S, updates the running max, computes P~ / 2^e per 32-key
//              block, quantizes it in registers, writes 64 bytes of codes (64B-swizzled, the MMA
//              operand layout) and four scale bytes to shared memory, rescales O and L in TMEM
//              when the max moves, and at the end normalises and stores the output row.
//   WS = 8     warps 4-11 tile A, 12-19 tile B (640 threads): two threads per query row, each
//              with one 64-key half of every key tile (a 16-lane, two-half tcgen05.ld), so that
//              each SM sub-partition runs four softmax warps; the row max and the conventional
//              row sum meet over one shuffle, everything else is per thread as above.
// TMEM (512 columns): S [0,128) O_A [128,128+d) O_B [256,256+d) L_A [384,400) L_B [400,416),
// scale atoms from 416 (see kColSf*).
// The kernel is templated on the format: MXFP4 (the method) or, for comparison, NVFP4 (blocks of
// 16 with E4M3 scales for Q, K, V and P~; kind::mxf4nvf4 products, the non-power-of-two P~ scale
// folded into the exponent bias as -log2 s), and on the rule that makes the P~ operand:
//   PM = 0  exp-then-quantize, row sum of the unquantized exponentials (the conventional path)
//   PM = 1  exp-then-quantize, row sum of the same quantized operand (PNQ)
//   PM = 2  exp-free codes (EFQ-Softmax abstract): per 32-key block the exponent-only scale of
//           the block max as above, then code k = clamp(round(2 r + 2), 0, 7) of the residual
//           r = S c - m c - e (the base-2 log of P~ / 2^e), no exponential per element; the row
//           sum again comes from the same operand. MXFP4 only.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "mxattn_internal.h"
#include "sm100_ptx.cuh"

namespace mxattn {

constexpr int kBM = 128;          // query rows per Q tile (the MMA's M)
constexpr int kBN = kKvTile;      // keys per KV tile (128)
// Two softmax layouts (the kernel's WS parameter, softmax warps per query tile):
//   WS = 4: one thread per query row, 384 threads (warpgroup 0 control, warpgroups 1-2 softmax).
//   WS = 8: two threads per query row (each a 64-key half of every key tile), 640 threads
//           (warpgroup 0 control, warpgroups 1-4 softmax): twice the warps on each SM
//           sub-partition to cover the softmax chain's waits, in half the registers per thread.
// Register split (per thread): the block is launched with kLaunchRegs (the ptxas limit for its
// thread count); warpgroup 0 gives back down to kCtlRegs, the softmax warpgroups grow to
// kSoftmaxRegs. The shares add up to exactly the launch total, which the host checks before
// launching.
template <int WS> struct Layout;
template <> struct Layout<4> {
  static constexpr int kThreads = 384, kLaunchRegs = 168, kCtlRegs = 88, kSoftmaxRegs = 208;
};
template <> struct Layout<8> {
  static constexpr int kThreads = 640, kLaunchRegs = 96, kCtlRegs = 64, kSoftmaxRegs = 104;
};
static_assert(128 * Layout<4>::kCtlRegs + 256 * Layout<4>::kSoftmaxRegs == Layout<4>::kThreads * Layout<4>::kLaunchRegs,
              "register split");
static_assert(128 * Layout<8>::kCtlRegs + 512 * Layout<8>::kSoftmaxRegs == Layout<8>::kThreads * Layout<8>::kLaunchRegs,
              "register split");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 128, kColL = 384;   // O_X at kColO + 128 X, L_X at kColL + 16 X
// Scale atoms, 4 columns each (NVFP4 needs two per operand tile, MXFP4 one):
//   Q_X         kColSfQ + 8 X
//   K of tile t kColSfK + 8 (t & 1)      V of tile t kColSfV + 8 (t & 1)
//   P~_X(t)     kColSfP + 16 X + 8 (t & 1)
//   ones        kColSf1 + 4 X (one copy per P~V issuer)
// tcgen05.cp into columns an earlier MMA still reads is not ordered behind that MMA; the K, V and
// P~ sets alternate by tile parity, and the set written for tile t was last read by a product of
// tile t - 2, which the copying thread has seen complete by then (see the S and P~V issuers).
constexpr uint32_t kColSfQ = 416, kColSfK = 432, kColSfV = 448, kColSfP = 464, kColSf1 = 496;   // + 4 x
constexpr int kOnesRows = 16;     // N of the row-sum MMA: row 0 all ones, rows 1..15 zero
constexpr int kPRowBytes = kBN / 2;                  // 64 bytes of codes per P~ / V^T row

static_assert(kBN == 128, "the 64B-swizzled P~ / V^T layouts below assume 128-key tiles");

template <int D>
struct Cfg {
  static constexpr int kStages = (D == 128) ? 6 : 8;
  static constexpr int kQRowBytes = D / 2;                 // packed E2M1 per Q/K row
  static constexpr int kQTileBytes = kBM * kQRowBytes;
  static constexpr int kKTileBytes = kBN * kQRowBytes;
  static constexpr int kVTileBytes = D * kPRowBytes;       // V^T: D rows of 128 keys
  static constexpr uint32_t kQKLayout = (D == 128) ? kLayoutSw64 : kLayoutSw32;
  static constexpr uint32_t kQKSbo = 8 * kQRowBytes;       // 8-row swizzle atom
};

template <int D>
struct __align__(1024) Smem {
  uint8_t q[2][Cfg<D>::kQTileBytes];
  uint8_t k[Cfg<D>::kStages][Cfg<D>::kKTileBytes];
  uint8_t v[Cfg<D>::kStages][Cfg<D>::kVTileBytes];
  uint8_t p[2][2][kBM * kPRowBytes];      // P~ codes [query tile][tile parity]
  uint8_t ones[kOnesRows * kPRowBytes];
  uint8_t qsf[2][1024];                   // per query tile: MXFP4 one atom, NVFP4 D / 64 atoms
  uint8_t ksf[Cfg<D>::kStages][1024];
  uint8_t vsf[Cfg<D>::kStages][1024];     // MXFP4 one atom per key tile, NVFP4 two
  uint8_t psf[2][2][1024];                // [query tile][tile parity]
  uint8_t onesf[512];
  uint64_t bar_q;
  uint64_t bar_kv_full[Cfg<D>::kStages];
  uint64_t bar_kv_empty[Cfg<D>::kStages];
  uint64_t bar_s_full[2];                 // S of query tile X computed (one phase per key tile)
  uint64_t bar_s_empty;                   // the S buffer's current user holds it in registers
  // P~ buffer [X][b] written by the four warps of query tile X (key tiles of parity b). One
  // barrier per buffer: a fast softmax warp may arrive for tile t+1 before a slow one has arrived
  // for tile t.
  uint64_t bar_p_full[2][2];
  uint64_t bar_pv_done[2][2];             // completions of PV of query tile X, even / odd key tiles
  uint64_t bar_drain[3];                  // each issuing warp's own final drain
  uint64_t bar_ones;                      // the ones operand is in shared memory (PNQ)
  uint32_t tmem_base;
  int abort_flag;
};

template <int D>
constexpr size_t smem_bytes() {
  return sizeof(Smem<D>) + 1024;
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

// 2^x on the FMA and ALU pipes, for a share of the PNQ exponentials that would otherwise queue on
// the MUFU. Only the E2M1 code of 2^x is kept, so the function has to fall on the correct side of
// every rounding midpoint of the grid (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5 times 2^e), not be
// accurate everywhere. Range reduction x = n + f with n = round(x), f in [-0.5, 0.5] (the
// 1.5 * 2^23 bias rounds to an integer in the mantissa); 2^f by the cubic through 2^f at
// f = log2 0.75, log2 0.875 and log2 1.25, with value 1 at f = 0 -- the four places where a
// midpoint of the grid falls after the reduction (log2 1.75 - 1 = log2 0.875). Between them the
// cubic is within 4e-4 of 2^f and increasing, which no code can see; at them it is within one
// fp32 ulp, like ex2.approx. The coefficients were fitted in fp64 and rounded to fp32. x is
// clamped at -127 so that n << 23 stays inside the exponent field (such values code to 0
// anyway).
__device__ __forceinline__ void exp2_codes_poly(float& y0, float& y1, float x0, float x1) {
  constexpr float kRound = 12582912.0f;                       // 1.5 * 2^23
  constexpr float kC1 = 0x1.630374p-1f, kC2 = 0x1.ee3f4ep-3f, kC3 = 0x1.b240f2p-5f;
  const float xc0 = fmaxf(x0, -127.f), xc1 = fmaxf(x1, -127.f);
  float t0, t1, n0, n1, f0, f1, p0, p1;
  fadd2(t0, t1, xc0, xc1, kRound, kRound);
  fadd2(n0, n1, t0, t1, -kRound, -kRound);
  fadd2(f0, f1, xc0, xc1, -n0, -n1);
  ffma2(p0, p1, f0, f1, kC3, kC3, kC2, kC2);
  ffma2(p0, p1, p0, p1, f0, f1, kC1, kC1);
  ffma2(p0, p1, p0, p1, f0, f1, 1.f, 1.f);
  y0 = __uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23));
  y1 = __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23));
}

// Wait of a whole warp for an mbarrier phase (bounded, see mbar_wait).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          unsigned int* status, unsigned int code) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, status, code));
}

// E8M0 byte of a P~ block maximum amax = 2^d in [0, 1] (the running max bounds every P~ by 1),
// read off d <= 0 itself, with no exponential: the OCP exponent floor(log2 amax) - 2 = floor(d) - 2,
// plus one under UOS when the significand 2^f, f = d - floor(d), exceeds 1.8125, i.e. when
// f > log2 1.8125 (0x1.b74948p-1 in fp32, whose 2^f is just below 1.8125). floor(d) comes from one
// round-down add of 1.5 * 2^23 (the sum's low mantissa bits then hold it) and f is exact. Every d
// below -126, d = -inf (an all-masked block) included, gives byte 0, as the general rule's clamp
// does for subnormal and zero maxima.
__device__ __forceinline__ uint32_t p_scale_byte_log2(float d, int mode) {
  constexpr float kMagic = 12582912.0f;                   // 1.5 * 2^23
  constexpr float kLog2UosLimit = 0x1.b74948p-1f;         // log2(1.8125) rounded to fp32
  const float dc = fmaxf(d, -160.f);
  const float t = __fadd_rd(dc, kMagic);                  // floor(dc) + 1.5 * 2^23, exactly
  const int e = __float_as_int(t) - 0x4B400000;           // floor(dc)
  const float f = dc - (t - kMagic);
  const int byte = e + 125 + ((mode == 1 && f > kLog2UosLimit) ? 1 : 0);
  return static_cast<uint32_t>(max(byte, 0));
}

// kPolyPairs of the 16 key pairs of every 32-key chunk take their PNQ exponentials from
// exp2_codes_poly (FMA and integer pipes) instead of the MUFU, spread evenly over the chunk. With
// the tcgen05 issue work spread over all four SM sub-partitions the softmax warps set the pace and
// the MUFU (16 results per clock per SM) is their busiest unit; measured on the video-DiT workload,
// 4, 5, 6 and 7 of 16 pairs gave +2%, +7%, +3% and +1% over none.
constexpr int kPolyPairs8 = 5, kPolyPairs16 = 3;   // one / two threads per row (WS = 4 / 8)
template <int kPolyPairs>
__host__ __device__ constexpr bool poly_pair(int pair) {
  return ((pair + 1) * kPolyPairs) / 16 > (pair * kPolyPairs) / 16;
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

// One thread's half of a row of D TMEM columns (D / 2 per thread, the halves 64 or 32 apart).
template <int D>
__device__ __forceinline__ void tmem_ld16x2_h(uint32_t taddr, uint32_t (&r)[D / 2]) {
  if constexpr (D == 128) tmem_ld16x2_64<64>(taddr, r);
  else tmem_ld16x2_32<32>(taddr, r);
}
template <int D>
__device__ __forceinline__ void tmem_st16x2_h(uint32_t taddr, const uint32_t (&r)[D / 2]) {
  if constexpr (D == 128) tmem_st16x2_64<64>(taddr, r);
  else tmem_st16x2_32<32>(taddr, r);
}

// NV = false: MXFP4 (blocks of 32, UE8M0, OCP or UOS exponent). NV = true: the NVFP4 comparison
// format for Q, K, V and P~ (blocks of 16, E4M3 scale = RNE(amax / 6)).
template <int D, int PM, bool DBG, bool NV, int WS>
__global__ void __launch_bounds__(Layout<WS>::kThreads, 1)
    mxattn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  static_assert(PM >= 0 && PM <= 2 && !(NV && PM == 2), "P~ rule");
  static_assert(WS == 4 || WS == 8, "softmax layout");
  constexpr int kCtlRegs = Layout<WS>::kCtlRegs, kSoftmaxRegs = Layout<WS>::kSoftmaxRegs;
  static_assert(offsetof(Smem<D>, p) % 1024 == 0 && sizeof(Smem<D>::p[0]) == 4 * 4096,
                "the output stage needs four 1024-aligned 4 KB quarters per query tile");
  constexpr bool PNQ = PM != 0;     // the row sum is the ones-operand product of the quantized P~
  constexpr bool EFQ = PM == 2;
  using C = Cfg<D>;
  constexpr int NS = C::kStages;
  constexpr int kQKAtoms = NV ? D / 64 : 1;            // scale atoms per 128 Q or K rows
  constexpr uint32_t kQKSfBytes = kQKAtoms * 512;
  constexpr int kPVAtoms = NV ? 2 : 1;                 // scale atoms per 128-key V^T or P~ tile
  constexpr uint32_t kPVSfBytes = kPVAtoms * 512;
  extern __shared__ uint8_t smem_raw[];
  Smem<D>& s = *reinterpret_cast<Smem<D>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work unit: (b, kv head g, query head within group, pair of q tiles). Non-causal: the pair
  //      index runs fastest, so that co-scheduled CTAs share one KV head in L2. Causal: units are
  //      ordered by length across all heads, longest first (the head index runs fastest, so that
  //      the CTAs in flight still cover few KV groups); the block scheduler's in-order dispatch then
  //      gives each SM the longest unit left, and the last wave holds the shortest ones.
  const int n_qt = p.Npad / kBM;
  const int n_units = (n_qt + 1) / 2;
  const int group = p.Hq / p.Hkv;
  const int n_bh = p.B * p.Hq;
  int unit, bh_q;
  if (p.causal) {
    unit = n_units - 1 - static_cast<int>(blockIdx.x / n_bh);
    bh_q = static_cast<int>(blockIdx.x % n_bh);
  } else {
    unit = static_cast<int>(blockIdx.x % n_units);
    bh_q = static_cast<int>(blockIdx.x / n_units);
  }
  const int b = bh_q / p.Hq;                  // bh_q = b * Hq + h  (h = g * group + hh)
  const int h = bh_q % p.Hq;
  const int bh_kv = b * p.Hkv + h / group;
  const int n_kv_all = p.Npad / kBN;
  int qt_x[2], n_kv_x[2];
#pragma unroll
  for (int x = 0; x < 2; ++x) {
    qt_x[x] = 2 * unit + x;
    n_kv_x[x] = qt_x[x] >= n_qt ? 0 : (p.causal ? min(qt_x[x] + 1, n_kv_all) : n_kv_all);
  }
  const bool has_b = n_kv_x[1] > 0;
  const int n_kv_max = max(n_kv_x[0], n_kv_x[1]);

  if (threadIdx.x == 0) {
    mbar_init(&s.bar_q, 1);
    for (int i = 0; i < NS; ++i) {
      mbar_init(&s.bar_kv_full[i], 1);
      mbar_init(&s.bar_kv_empty[i], 2);    // one release per P~V issuer
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&s.bar_s_full[x], 1);
      for (int i = 0; i < 2; ++i) {
        mbar_init(&s.bar_p_full[x][i], WS);     // one arrival per softmax warp of the tile
        mbar_init(&s.bar_pv_done[x][i], 1);
      }
    }
    mbar_init(&s.bar_s_empty, WS);
    for (int i = 0; i < 3; ++i) mbar_init(&s.bar_drain[i], 1);
    mbar_init(&s.bar_ones, 1);
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

  if (warp < 4) {
   regs_dec<kCtlRegs>();
   // Four control warps, one per SM sub-partition: warp 2 the TMA loads, warp 1 the S products
   // (the latency-critical hand-overs of the S buffer), warps 0 and 3 the P~V and row-sum
   // products of tiles A and B. Each waits on the barriers that gate its own work; the
   // scale-atom sets stay safe as argued beside each copy below.
   const uint64_t sf_desc_base = smem_desc(0, 0, 128, kLayoutNone);
   auto sf_desc = [&](const void* ptr) { return sf_desc_base | ((smem_u32(ptr) >> 4) & 0x3FFFu); };
   // Shared-memory descriptors: only the 14-bit start-address field (16-byte units) differs between
   // the operands of one kind, so each is one OR of a fixed upper part with an address.
   const uint64_t d_qk = smem_desc(0, 0, C::kQKSbo, C::kQKLayout);          // Q and K tiles
   const uint64_t d_pv = smem_desc(0, 0, 8 * kPRowBytes, kLayoutSw64);      // P~, V^T and ones tiles
   const uint32_t a_q = smem_u32(s.q[0]) >> 4, a_k = smem_u32(s.k[0]) >> 4, a_v = smem_u32(s.v[0]) >> 4;
   const uint32_t a_p = smem_u32(s.p[0][0]) >> 4, a_ones = smem_u32(s.ones) >> 4;
   if (warp == 2) {
    // ============================ TMA producer ============================
    // The whole warp runs the loop (warp-uniform operands); one elected lane issues the copies.
    const bool leader = elect_one_sync();
    if (leader) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      mbar_arrive_expect_tx(&s.bar_q, (has_b ? 2u : 1u) * (C::kQTileBytes + kQKSfBytes));
      for (int x = 0; x < (has_b ? 2 : 1); ++x) {
        tma_load_2d(s.q[x], &tmQ, &s.bar_q, 0, bh_q * p.rows_per_head + qt_x[x] * kBM);
        bulk_load(s.qsf[x], p.qsf + (static_cast<size_t>(bh_q) * n_qt + qt_x[x]) * kQKSfBytes, kQKSfBytes,
                  &s.bar_q);
      }
    }
    __syncwarp();
    int issued = 0;
    for (int t = 0; t < n_kv_max; ++t) {
      const int st = t % NS;
      if (t >= NS &&
          !warp_wait(&s.bar_kv_empty[st], ((t / NS) & 1) ^ 1, abort_flag, p.status, kStatusTimeoutEmpty | st))
        break;
      if (leader) {
        mbar_arrive_expect_tx(&s.bar_kv_full[st], C::kKTileBytes + C::kVTileBytes + kQKSfBytes + kPVSfBytes);
        tma_load_2d(s.k[st], &tmK, &s.bar_kv_full[st], 0, bh_kv * p.rows_per_head + t * kBN);
        tma_load_2d(s.v[st], &tmV, &s.bar_kv_full[st], t * kPRowBytes, bh_kv * D);
        bulk_load(s.ksf[st], p.ksf + (static_cast<size_t>(bh_kv) * n_qt + t) * kQKSfBytes, kQKSfBytes,
                  &s.bar_kv_full[st]);
        // V^T atoms: MXFP4 one per 128 keys; NVFP4 one per 64 keys, two per key tile
        const size_t v_at = NV ? static_cast<size_t>(bh_kv) * (p.Npad / 64) + 2 * t
                               : static_cast<size_t>(bh_kv) * n_qt + t;
        bulk_load(s.vsf[st], p.vsf + v_at * 512, kPVSfBytes, &s.bar_kv_full[st]);
      }
      __syncwarp();
      issued = t + 1;
    }
    if (*abort_flag && leader) {
      // let every copy this warp started land before the CTA can exit
      drain_wait(&s.bar_q, 0);
      for (int t = (issued > NS ? issued - NS : 0); t < issued; ++t)
        drain_wait(&s.bar_kv_full[t % NS], (t / NS) & 1);
    }
    __syncwarp();
   } else if (warp == 0 || warp == 3) {
    // ======================= P~V issuer of query tile x (warp 0: A, warp 3: B) =======================
    // One elected thread copies the P~ (and, for the first product of a key tile, the V) scale atoms
    // to TMEM and issues O_x += P~_x(t) V(t) and L_x += P~_x(t) 1 once tile x's softmax hands P~
    // over. A commit arrives only when every earlier operation of its thread has completed.
    const int x = warp == 0 ? 0 : 1;
    const bool leader = elect_one_sync();
    const uint32_t ones_sf = tmem + kColSf1 + 4 * x;      // each issuer holds its own ones atom
    if (PNQ) {
      if (x == 0) {
        // ones operand (row 0 = code 1.0 for every key, rows 1..15 = 0) with unit scales
        uint32_t* ow = reinterpret_cast<uint32_t*>(s.ones);
        for (int i = lane; i < kOnesRows * kPRowBytes / 4; i += 32) ow[i] = (i < kPRowBytes / 4) ? 0x22222222u : 0u;
        uint32_t* sw = reinterpret_cast<uint32_t*>(s.onesf);
        for (int i = lane; i < 512 / 4; i += 32) sw[i] = NV ? 0x38383838u : 0x7F7F7F7Fu;   // E4M3 / E8M0 1.0
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.bar_ones);
      }
      bool ok1 = warp_wait(&s.bar_ones, 0, abort_flag, p.status, kStatusTimeoutQ | 1);
      tc_fence_after();
      if (ok1 && leader) tc_cp_sf(ones_sf, sf_desc(s.onesf));
      __syncwarp();
    }
    const int n_own = x == 0 ? n_kv_x[0] : n_kv_x[1];
    const int n_other = x == 0 ? n_kv_x[1] : n_kv_x[0];
    bool ok = true;
    for (int t = 0; ok && t < n_kv_max; ++t) {
      const int st = t % NS;
      const int pb = t & 1;
      // no product of this query tile reads key tile t: the other issuer releases the stage for
      // both (an issuer that arrived here on its own could run ahead and arrive twice on one phase)
      if (t >= n_own) continue;
      ok = warp_wait(&s.bar_p_full[x][pb], (t >> 1) & 1, abort_flag, p.status, kStatusTimeoutP);
      if (!ok) break;
      // The V scale atoms of key tile t are copied by its first product: PV(A, t), or PV(B, t) when
      // tile A has no product there. The other issuer's PV(t) waits for that product (its commit
      // covers the copy). Before the copy, the set's last readers PV(., t - 2) must be complete:
      // this issuer's own was seen complete by its softmax (which reused the P~ buffer after it),
      // the other issuer's is waited for here.
      const bool first = (x == 0) || t >= n_other;
      if (!first) {
        ok = warp_wait(&s.bar_pv_done[0][pb], (t >> 1) & 1, abort_flag, p.status, kStatusTimeoutPV | 2);
      } else if (t >= 2 && t - 2 < n_other) {
        ok = warp_wait(&s.bar_pv_done[x ^ 1][pb], ((t >> 1) - 1) & 1, abort_flag, p.status,
                            kStatusTimeoutPV | 3);
      }
      if (!ok) break;
      tc_fence_after();
      if (leader) {
        const uint32_t sfp = tmem + kColSfP + 16 * x + 8 * pb;
        const uint32_t sfv = tmem + kColSfV + 8 * pb;
#pragma unroll
        for (int a = 0; a < kPVAtoms; ++a) tc_cp_sf(sfp + 4 * a, sf_desc(s.psf[x][pb] + a * 512));
        if (first) {
#pragma unroll
          for (int a = 0; a < kPVAtoms; ++a) tc_cp_sf(sfv + 4 * a, sf_desc(s.vsf[st] + a * 512));
        }
        const uint32_t o_col = tmem + kColO + 128 * x, l_col = tmem + kColL + 16 * x;
        const uint32_t pa = a_p + (2 * x + pb) * ((kBM * kPRowBytes) >> 4), va = a_v + st * (C::kVTileBytes >> 4);
#pragma unroll
        for (int kk = 0; kk < kBN / 64; ++kk) {
          const uint64_t ad = d_pv | (pa + kk * 2), bd = d_pv | (va + kk * 2), od = d_pv | (a_ones + kk * 2);
          const uint32_t acc = (t > 0 || kk > 0) ? 1u : 0u;
          if constexpr (NV) {
            tc_mma_nvf4(o_col, ad, bd, idesc_nvf4(D), sfp + 4 * kk, sfv + 4 * kk, acc);
            if (PNQ) tc_mma_nvf4(l_col, ad, od, idesc_nvf4(kOnesRows), sfp + 4 * kk, ones_sf, acc);
          } else {
            // keys 64 kk .. 64 kk + 63 are blocks 2 kk, 2 kk + 1 of the P~ and V^T scale atoms
            tc_mma_mxf4(o_col, ad, bd, idesc_mxf4(D, 2 * kk, 2 * kk), sfp, sfv, acc);
            if (PNQ) tc_mma_mxf4(l_col, ad, od, idesc_mxf4(kOnesRows, 2 * kk, 0), sfp, ones_sf, acc);
          }
        }
        tc_commit(&s.bar_pv_done[x][pb]);
        // this issuer's release of the stage: the S products that read its K tile were complete
        // before this product's softmax could read S(x, t). When the other tile has no product at
        // key tile t, the second arrival is made here too; the phase still completes only with
        // the commit.
        tc_commit(&s.bar_kv_empty[st]);
        if (t >= n_other) mbar_arrive(&s.bar_kv_empty[st]);
      }
      __syncwarp();
    }
    // every product / copy issued above must complete before TMEM is released
    if (leader) {
      tc_commit(&s.bar_drain[x]);
      drain_wait(&s.bar_drain[x], 0);
    }
    __syncwarp();
   } else if (warp == 1) {
    // ======================= TMEM owner and S issuer =======================
    // Order: S(A, t), S(B, t), S(A, t+1), ...: each waits until the previous user of the S buffer
    // holds its scores in registers. A commit arrives only when every earlier operation of this
    // thread has completed, so when this thread has seen the user of S(., t - 1) read it, the S
    // products of tile t - 2 are complete: the K set of tile t, which they read, may be rewritten
    // (before that wait: the wait that S(., t - 1) itself passed already implies it).
    const bool leader = elect_one_sync();
    bool ok = warp_wait(&s.bar_q, 0, abort_flag, p.status, kStatusTimeoutQ);
    if (ok) {
      tc_fence_after();
      if (leader) {
        for (int x = 0; x < (has_b ? 2 : 1); ++x) {
#pragma unroll
          for (int a = 0; a < kQKAtoms; ++a) tc_cp_sf(tmem + kColSfQ + 8 * x + 4 * a, sf_desc(s.qsf[x] + a * 512));
        }
      }
      __syncwarp();
    }
    int s_uses = 0;      // S products issued so far (A and B alternate on the one buffer)
    auto issue_s = [&](int x, int t) -> bool {
      const int st = t % NS;
      const bool first = (x == 0) || t >= n_kv_x[0];      // first product of key tile t
      const uint32_t sfk = tmem + kColSfK + 8 * (t & 1);
      if (first) {
        if (!warp_wait(&s.bar_kv_full[st], (t / NS) & 1, abort_flag, p.status, kStatusTimeoutKV | st))
          return false;
        tc_fence_after();
        if (leader) {
#pragma unroll
          for (int a = 0; a < kQKAtoms; ++a) tc_cp_sf(sfk + 4 * a, sf_desc(s.ksf[st] + a * 512));
        }
      }
      // the previous user of the S buffer must hold its scores in registers
      if (s_uses > 0 &&
          !warp_wait(&s.bar_s_empty, (s_uses - 1) & 1, abort_flag, p.status, kStatusTimeoutS))
        return false;
      // tile x's softmax writes P~(x, t) into the buffer that P~V(x, t - 2) read: that product must be
      // complete before S(x, t) is handed over (it is, long since, in the steady state; waiting here
      // keeps the wait off the softmax warps' path)
      if (t >= 2 && !warp_wait(&s.bar_pv_done[x][t & 1], ((t >> 1) - 1) & 1, abort_flag, p.status, kStatusTimeoutPV))
        return false;
      tc_fence_after();
      if (leader) {
        const uint32_t qa = a_q + x * (C::kQTileBytes >> 4), ka = a_k + st * (C::kKTileBytes >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 64; ++kk) {
          const uint64_t ad = d_qk | (qa + kk * 2), bd = d_qk | (ka + kk * 2);   // +32 bytes per K = 64
          if constexpr (NV)   // one atom (four 16-element blocks) per K = 64 step
            tc_mma_nvf4(tmem + kColS, ad, bd, idesc_nvf4(kBN), tmem + kColSfQ + 8 * x + 4 * kk, sfk + 4 * kk, kk > 0);
          else
            tc_mma_mxf4(tmem + kColS, ad, bd, idesc_mxf4(kBN, 2 * kk, 2 * kk), tmem + kColSfQ + 8 * x, sfk, kk > 0);
        }
        tc_commit(&s.bar_s_full[x]);
      }
      __syncwarp();
      ++s_uses;
      return true;
    };
    if (ok && n_kv_x[0] > 0) ok = issue_s(0, 0);
    if (ok && n_kv_x[1] > 0) ok = issue_s(1, 0);
    for (int t = 0; ok && t + 1 < n_kv_max; ++t) {
      if (ok && t + 1 < n_kv_x[0]) ok = issue_s(0, t + 1);
      if (ok && t + 1 < n_kv_x[1]) ok = issue_s(1, t + 1);
    }
    // every product / copy issued above must complete before TMEM is released
    if (leader) {
      tc_commit(&s.bar_drain[2]);
      drain_wait(&s.bar_drain[2], 0);
    }
    __syncwarp();
   }
  } else {
    regs_inc<kSoftmaxRegs>();
    if constexpr (WS == 8) {

      // ============================ softmax warps ============================
      // Two threads per query row: eight warps per tile, two per TMEM lane quarter (16 rows each).
      // Thread (lane & 15) of a warp owns row r of its 16 and keys [64 kh, 64 kh + 64) of each key
      // tile (kh = lane >> 4): the 16-lane, two-half TMEM load gives each half-warp the same lanes
      // at columns 64 apart. The row max and the conventional row sum meet over one shuffle with
      // the partner thread (lane ^ 16); block maxima, scale bytes and P~ codes stay thread-local.
      const int sw = warp - 4;
      const int x = sw >> 3;                            // query tile: warps 4-11 A, 12-19 B
      const int hh = (sw >> 2) & 1;                     // which 16 rows of the lane quarter
      const int quarter = warp & 3;                     // TMEM lane quarter this warp may access
      const int kh = lane >> 4;                         // key half of the tile (and of O's columns)
      const int r0 = quarter * 32 + hh * 16;            // first row of this warp
      const int r = r0 + (lane & 15);                   // row inside the tile == TMEM lane
      const int qt = x == 0 ? qt_x[0] : qt_x[1];
      const int n_kv = x == 0 ? n_kv_x[0] : n_kv_x[1];
      const int qrow = qt * kBM + r;
      const uint32_t lane_addr = static_cast<uint32_t>(r0) << 16;
      const uint32_t o_col = tmem + lane_addr + kColO + 128 * x;
      const uint32_t l_col = tmem + lane_addr + kColL + 16 * x;
      const float c = p.scale_log2;
      constexpr int kPB = NV ? 16 : 32;                 // keys per P~ scale block
      constexpr int kNPB = kBN / kPB;                   // scale blocks per row per tile
      constexpr int kNPBt = kNPB / 2;                   // ... of which this thread owns
      constexpr int kHalf = kBN / 2;                    // keys per thread per tile
      const float c27 = c * (2.f / 7.f);                // exp-free rule: (2 r + 2) / 7 = S c27 + b7
      float m = -INFINITY;      // running max of the raw scores S
      float l = 0.f;            // running row sum (pnq = 0), this thread's half
      bool ok = n_kv > 0;
      const bool dbg = DBG && bh_q == p.dbg_bh && qrow >= p.dbg_r0 && qrow < p.dbg_r1;
      const uint32_t swz = (static_cast<uint32_t>(r) >> 1) & 3u;   // 64-byte swizzle of this row
      const uint32_t psf_off = (r & 31) * 16 + (r >> 5) * 4;

      for (int t = 0; ok && t < n_kv; ++t) {
        ok = warp_wait(&s.bar_s_full[x], t & 1, abort_flag, p.status, kStatusTimeoutS | 8);
        if (!ok) break;
        tc_fence_after();
        float sv[kHalf];
        {
          uint32_t raw[kHalf];
          tmem_ld16x2_64<kHalf>(tmem + lane_addr + kColS, raw);
          tc_wait_ld();
#pragma unroll
          for (int i = 0; i < kHalf; ++i) sv[i] = __uint_as_float(raw[i]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.bar_s_empty);

        // masking: keys beyond N, and keys after the query row when causal
        const int key0 = t * kBN + kh * kHalf;
        if (t * kBN + kBN > p.N || (p.causal && t * kBN + kBN - 1 > qt * kBM)) {
          const int lim = (p.causal ? min(p.N, qrow + 1) : p.N) - key0;   // keys [key0, key0 + lim) count
#pragma unroll
          for (int i = 0; i < kHalf; ++i) sv[i] = (i < lim) ? sv[i] : -INFINITY;
        }
        float bmax[kNPBt];
#pragma unroll
        for (int bb = 0; bb < kNPBt; ++bb) bmax[bb] = NV ? block_max16(sv + bb * kPB) : block_max32(sv + bb * kPB);
        float tmax = bmax[0];
#pragma unroll
        for (int bb = 1; bb < kNPBt; ++bb) tmax = fmaxf(tmax, bmax[bb]);
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 16));
        const float m_new = fmaxf(m, tmax);
        const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
        // the history factor alpha = 2^((m - m') c) only where some row of the warp saw its max move
        // (elsewhere it is 1); it is read by the rescale below and by the conventional row sum
        const bool moved = __any_sync(0xffffffffu, m_new > m);
        float alpha = 1.f;
        if (moved) alpha = (m == -INFINITY) ? 0.f : ex2_approx((m - m_use) * c);

        uint32_t sbytes = 0;      // this thread's scale bytes, block order
        float nb[kNPBt], bscale[kNPBt];
#pragma unroll
        for (int bb = 0; bb < kNPBt; ++bb) {
          uint32_t byte;
          if constexpr (NV) {
            const float amax = ex2_approx((bmax[bb] - m_use) * c);   // 0 for an all-masked block
            // s = E4M3(amax / 6), the quotient as amax times fp32(1/6): within one ulp of the
            // correctly rounded quotient, so the E4M3 rounding can only differ where the quotient
            // lies within an ulp of one of its midpoints (amax itself comes from ex2.approx). s = 0
            // (amax <= 6 * 2^-10): y = P~ itself (every value below the 0.25 rounding threshold,
            // so the codes are 0 as the format wants) and the unquantized row sum still counts the
            // block with weight 1
            byte = e4m3_byte(amax * (1.0f / 6.0f));
            const float sb = e4m3_value(byte);
            bscale[bb] = sb > 0.f ? sb : 1.f;
            nb[bb] = sb > 0.f ? fmaf(-m_use, c, -lg2_approx(sb)) : -m_use * c;
          } else {
            // the byte of amax = 2^((bmax - m') c) straight from the exponent (no MUFU on this path)
            byte = p_scale_byte_log2((bmax[bb] - m_use) * c, p.mode);
            // 127 - byte as a float without a conversion: it sits in the low mantissa bits of 2^23
            const float neg_e = __uint_as_float(0x4B000000u + (127u - byte)) - 8388608.0f;
            nb[bb] = fmaf(-m_use, c, neg_e);
            bscale[bb] = pow2_from_byte(byte);
          }
          sbytes |= byte << (8 * bb);
        }
        // P~ buffer t&1: its last reader, the product of key tile t-2, completed before S(x, t) was
        // issued (the S issuer waits for it)
        const int pb = t & 1;
        // 32 keys at a time (this thread's two 16-byte pieces of the row)
        uint8_t* p_row = s.p[x][pb] + r * kPRowBytes;
        uint8_t* d_row = (DBG && dbg) ? p.dbg_codes + static_cast<size_t>(qrow - p.dbg_r0) * (p.Npad / 2) + t * kPRowBytes
                                      : nullptr;
        float tile_sum = 0.f;
#pragma unroll
        for (int cc = 0; cc < kHalf / 32; ++cc) {
          const int jc = kh * (kHalf / 32) + cc;          // 16-byte piece of the row
          float* y = sv + 32 * cc;
          uint4 w4;
          if constexpr (EFQ) {
            // w = sat((2 r + 2) / 7); w times 7 * 2^-149 lands on the subnormal grid, so the product's
            // bit pattern is round(7 w) in [0, 7] (round to nearest even): the code itself
            const float b7 = fmaf(nb[cc], 2.f / 7.f, 2.f / 7.f);
            uint32_t wd[4];
#pragma unroll
            for (int w = 0; w < 4; ++w) {
              float k[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) k[i] = fma_sat(y[8 * w + i], c27, b7);
#pragma unroll
              for (int i = 0; i < 8; i += 2) fmul2_b(k[i], k[i + 1], k[i], k[i + 1], __uint_as_float(7u));
              uint32_t acc = pack_u4x2(0u, __float_as_uint(k[7]), __float_as_uint(k[6]));
              acc = pack_u4x2(acc, __float_as_uint(k[5]), __float_as_uint(k[4]));
              acc = pack_u4x2(acc, __float_as_uint(k[3]), __float_as_uint(k[2]));
              wd[w] = pack_u4x2(acc, __float_as_uint(k[1]), __float_as_uint(k[0]));
            }
            w4 = make_uint4(wd[0], wd[1], wd[2], wd[3]);
          } else {
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
              float x0, x1;
              ffma2_bc(x0, x1, y[i], y[i + 1], c, nb[(32 * cc + i) / kPB]);
              if (PM == 1 && poly_pair<kPolyPairs16>(i / 2)) {
                exp2_codes_poly(y[i], y[i + 1], x0, x1);
              } else {
                y[i] = ex2_approx_ftz(x0);
                y[i + 1] = ex2_approx_ftz(x1);
              }
            }
            w4 = make_uint4(cvt_e2m1x8(y), cvt_e2m1x8(y + 8), cvt_e2m1x8(y + 16), cvt_e2m1x8(y + 24));
          }
          *reinterpret_cast<uint4*>(p_row + ((static_cast<uint32_t>(jc) ^ swz) << 4)) = w4;
          if (DBG && dbg) reinterpret_cast<uint4*>(d_row)[jc] = w4;
          if (!PNQ) {   // conventional row sum of the unquantized exponentials
#pragma unroll
            for (int bb = 0; bb < 32 / kPB; ++bb) {
              float b0 = 0.f, b1 = 0.f;
#pragma unroll
              for (int i = 0; i < kPB; i += 2) {
                b0 += y[bb * kPB + i];
                b1 += y[bb * kPB + i + 1];
              }
              tile_sum = fmaf(b0 + b1, bscale[(32 * cc) / kPB + bb], tile_sum);
            }
          }
        }
        if (!PNQ) l = fmaf(alpha, l, tile_sum);
        if constexpr (NV)   // two atoms per tile (keys 0-63, 64-127), four blocks each
          *reinterpret_cast<uint32_t*>(s.psf[x][pb] + kh * 512 + psf_off) = sbytes;
        else                // one atom, this thread's two of its four blocks
          *reinterpret_cast<uint16_t*>(s.psf[x][pb] + psf_off + 2 * kh) = static_cast<uint16_t>(sbytes);
        if (DBG && dbg) {
          uint8_t* ds = p.dbg_scales + static_cast<size_t>(qrow - p.dbg_r0) * (p.Npad / kPB) + t * kNPB + kh * kNPBt;
#pragma unroll
          for (int bb = 0; bb < kNPBt; ++bb) ds[bb] = static_cast<uint8_t>(sbytes >> (8 * bb));
        }
        fence_proxy_async_smem();

        // history rescale of O and L (only when some row of this warp saw its max move); O may only
        // be touched once the product of key tile t-1 has landed in it
        if (t > 0 && moved) {
          ok = warp_wait(&s.bar_pv_done[x][pb ^ 1], ((t - 1) >> 1) & 1, abort_flag, p.status, kStatusTimeoutPV | 4);
          if (!ok) break;
          tc_fence_after();
          {
            // this thread's half of O's columns, and L in the 16-lane x 2-column layout (thread t
            // holds row (t >> 2) + 8 (t & 1) of the 16, whose alpha its row owner passes over)
            uint32_t raw[D / 2];
            tmem_ld16x2_h<D>(o_col, raw);
            const uint32_t lv = PNQ ? tmem_ld16x64b_1(l_col) : 0u;
            const float alpha_l = __shfl_sync(0xffffffffu, alpha, ((lane >> 2) + 8 * (lane & 1)));
            tc_wait_ld();
#pragma unroll
            for (int i = 0; i < D / 2; i += 2) {
              float o0, o1;
              fmul2_b(o0, o1, __uint_as_float(raw[i]), __uint_as_float(raw[i + 1]), alpha);
              raw[i] = __float_as_uint(o0);
              raw[i + 1] = __float_as_uint(o1);
            }
            tmem_st16x2_h<D>(o_col, raw);
            if (PNQ) tmem_st16x64b_1(l_col, __float_as_uint(__uint_as_float(lv) * alpha_l));
          }
          tc_wait_st();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.bar_p_full[x][pb]);
        m = m_new;
      }

      // ---- epilogue: out = O / l (PV products complete in order: the last one covers all)
      if (ok) {
        ok = warp_wait(&s.bar_pv_done[x][(n_kv - 1) & 1], ((n_kv - 1) >> 1) & 1, abort_flag, p.status,
                       kStatusTimeoutPV | 1);
      }
      if (ok) {
        tc_fence_after();
        if (PNQ) {
          uint32_t lv[1];
          tmem_ld16x2_1<0>(l_col, lv);        // both halves read the row's sum in column 0
          tc_wait_ld();
          l = __uint_as_float(lv[0]);
        } else {
          l += __shfl_xor_sync(0xffffffffu, l, 16);
        }
        const float inv_l = 1.f / l;
        // The normalised rows leave through shared memory so that the global writes are whole lines:
        // per round, a 16-row x 128-byte stage (this warp's rows of the tile's two P~ buffers, which
        // no product reads any more) takes the 128 bytes of each row that the round covers, written
        // by the thread of the row that holds them, then the warp reads it back line-wise (eight
        // lanes per line) and stores it. 128-byte swizzle: the 16-byte piece j of stage row rr sits
        // at position j ^ (rr & 7). fp32: a round is 32 columns, bf16 64.
        auto stage_row = [&](int rr) {
          return smem_u32(s.p[x][rr >> 3]) + static_cast<uint32_t>(r0 + 2 * (rr & 7)) * kPRowBytes;
        };
        const int es = p.out_bf16 ? 2 : 4;
        const int rounds = D * es / 128;
        const int y0 = qt * kBM + r0;
        uint8_t* const ohead = static_cast<uint8_t*>(p.out) + static_cast<size_t>(bh_q) * p.N * D * es;
        const uint32_t my_row = stage_row(lane & 15);
        const uint32_t rsw = static_cast<uint32_t>(lane) & 7u;
#pragma unroll 1
        for (int g = 0; g < rounds; ++g) {
          if (p.out_bf16) {
            // round g: columns [64 g, 64 g + 64); with D = 128 one half's whole range (half g),
            // with D = 64 32 columns from each half
            uint32_t ov[32];
            tmem_ld16x2_32<D / 2>(o_col + (D == 128 ? 32u * 0u : 0u), ov);   // first 32 of each half
            uint32_t ow[32];
            tmem_ld16x2_32<D / 2>(o_col + (D == 128 ? 32u : 0u), ow);        // next 32 (D = 128)
            tc_wait_ld();
            const bool mine = (D == 128) ? (kh == g) : true;
            if (mine) {
#pragma unroll
              for (int pc = 0; pc < (D == 128 ? 8 : 4); ++pc) {
                uint32_t w[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                  const int i = 8 * pc + 2 * u;
                  const float a0 = __uint_as_float(i < 32 ? ov[i & 31] : ow[i & 31]) * inv_l;
                  const float a1 = __uint_as_float(i + 1 < 32 ? ov[(i + 1) & 31] : ow[(i + 1) & 31]) * inv_l;
                  const __nv_bfloat162 h2 = __floats2bfloat162_rn(a0, a1);
                  w[u] = *reinterpret_cast<const uint32_t*>(&h2);
                }
                const int piece = (D == 128) ? pc : 4 * kh + pc;
                st_shared_v4(my_row + ((static_cast<uint32_t>(piece) ^ rsw) << 4), w[0], w[1], w[2], w[3]);
              }
            }
          } else {
            // round g: columns [32 g, 32 g + 32), held by half g / (D / 64) at its offset 32 (g % (D / 64))
            uint32_t ov[32];
            tmem_ld16x2_32<D / 2>(o_col + 32u * static_cast<uint32_t>(g % (D / 64)), ov);
            tc_wait_ld();
            if (kh == g / (D / 64)) {
#pragma unroll
              for (int pc = 0; pc < 8; ++pc)
                st_shared_v4(my_row + ((static_cast<uint32_t>(pc) ^ rsw) << 4),
                             __float_as_uint(__uint_as_float(ov[4 * pc]) * inv_l),
                             __float_as_uint(__uint_as_float(ov[4 * pc + 1]) * inv_l),
                             __float_as_uint(__uint_as_float(ov[4 * pc + 2]) * inv_l),
                             __float_as_uint(__uint_as_float(ov[4 * pc + 3]) * inv_l));
            }
          }
          __syncwarp();
#pragma unroll
          for (int it = 0; it < 4; ++it) {
            const int idx = it * 32 + lane;
            const int rr = idx >> 3, pc = idx & 7;
            const uint4 val = ld_shared_v4(stage_row(rr) + ((static_cast<uint32_t>(pc) ^ (static_cast<uint32_t>(rr) & 7u)) << 4));
            if (y0 + rr < p.N)
              *reinterpret_cast<uint4*>(ohead + static_cast<size_t>(y0 + rr) * D * es + g * 128 + pc * 16) = val;
          }
          __syncwarp();     // the stage is read before the next round overwrites it
        }
      }
      tc_fence_before();
    } else {

      // ============================ softmax warps ============================
      const int x = (warp - 4) >> 2;                    // query tile: warps 4-7 A, 8-11 B
      const int quarter = warp & 3;                     // TMEM lane quarter this warp may access
      const int r = quarter * 32 + lane;                // row inside the tile == TMEM lane
      const int qt = x == 0 ? qt_x[0] : qt_x[1];
      const int n_kv = x == 0 ? n_kv_x[0] : n_kv_x[1];
      const int qrow = qt * kBM + r;
      const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
      const uint32_t o_col = tmem + lane_addr + kColO + 128 * x;
      const uint32_t l_col = tmem + lane_addr + kColL + 16 * x;
      const float c = p.scale_log2;
      constexpr int kPB = NV ? 16 : 32;                 // keys per P~ scale block
      constexpr int kNPB = kBN / kPB;                   // scale blocks per row per tile
      const float c27 = c * (2.f / 7.f);                // exp-free rule: (2 r + 2) / 7 = S c27 + b7
      float m = -INFINITY;      // running max of the raw scores S
      float l = 0.f;            // running row sum (pnq = 0)
      bool ok = n_kv > 0;
      const bool dbg = DBG && bh_q == p.dbg_bh && qrow >= p.dbg_r0 && qrow < p.dbg_r1;
      const uint32_t swz = (static_cast<uint32_t>(r) >> 1) & 3u;   // 64-byte swizzle of this row
      const uint32_t psf_off = (r & 31) * 16 + (r >> 5) * 4;

      for (int t = 0; ok && t < n_kv; ++t) {
        ok = warp_wait(&s.bar_s_full[x], t & 1, abort_flag, p.status, kStatusTimeoutS | 8);
        if (!ok) break;
        tc_fence_after();
        float sv[kBN];
        {
          uint32_t raw[kBN];
#pragma unroll
          for (int cc = 0; cc < kBN / 32; ++cc)
            tmem_ld32(tmem + lane_addr + kColS + 32 * cc, *reinterpret_cast<uint32_t(*)[32]>(raw + 32 * cc));
          tc_wait_ld();
#pragma unroll
          for (int i = 0; i < kBN; ++i) sv[i] = __uint_as_float(raw[i]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.bar_s_empty);

        // masking: keys beyond N, and keys after the query row when causal
        const int key0 = t * kBN;
        if (key0 + kBN > p.N || (p.causal && key0 + kBN - 1 > qt * kBM)) {
          const int lim = (p.causal ? min(p.N, qrow + 1) : p.N) - key0;   // keys [key0, key0 + lim) count
#pragma unroll
          for (int i = 0; i < kBN; ++i) sv[i] = (i < lim) ? sv[i] : -INFINITY;
        }
        // per block (32 keys for MXFP4, 16 for NVFP4): amax from the exact difference (1 for the
        // block that holds the max), the block's scale byte, and the exponent bias nb of
        // y = P~ / s = 2^(S c - m c - log2 s): one packed FMA per two elements and one ex2 each
        float bmax[kNPB];
#pragma unroll
        for (int bb = 0; bb < kNPB; ++bb) bmax[bb] = NV ? block_max16(sv + bb * kPB) : block_max32(sv + bb * kPB);
        float tmax = bmax[0];
#pragma unroll
        for (int bb = 1; bb < kNPB; ++bb) tmax = fmaxf(tmax, bmax[bb]);
        const float m_new = fmaxf(m, tmax);
        const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
        // the history factor alpha = 2^((m - m') c) only where some row of the warp saw its max move
        // (elsewhere it is 1); it is read by the rescale below and by the conventional row sum
        const bool moved = __any_sync(0xffffffffu, m_new > m);
        float alpha = 1.f;
        if (moved) alpha = (m == -INFINITY) ? 0.f : ex2_approx((m - m_use) * c);

        uint32_t sbytes[kNPB / 4];
        float nb[kNPB], bscale[kNPB];
#pragma unroll
        for (int bb = 0; bb < kNPB; ++bb) {
          uint32_t byte;
          if constexpr (NV) {
            const float amax = ex2_approx((bmax[bb] - m_use) * c);   // 0 for an all-masked block
            // s = E4M3(amax / 6), the quotient as amax times fp32(1/6): within one ulp of the
            // correctly rounded quotient, so the E4M3 rounding can only differ where the quotient
            // lies within an ulp of one of its midpoints (amax itself comes from ex2.approx). s = 0
            // (amax <= 6 * 2^-10): y = P~ itself (every value below the 0.25 rounding threshold,
            // so the codes are 0 as the format wants) and the unquantized row sum still counts the
            // block with weight 1
            byte = e4m3_byte(amax * (1.0f / 6.0f));
            const float sb = e4m3_value(byte);
            bscale[bb] = sb > 0.f ? sb : 1.f;
            nb[bb] = sb > 0.f ? fmaf(-m_use, c, -lg2_approx(sb)) : -m_use * c;
          } else {
            // the byte of amax = 2^((bmax - m') c) straight from the exponent (no MUFU on this path)
            byte = p_scale_byte_log2((bmax[bb] - m_use) * c, p.mode);
            // 127 - byte as a float without a conversion: it sits in the low mantissa bits of 2^23
            const float neg_e = __uint_as_float(0x4B000000u + (127u - byte)) - 8388608.0f;
            nb[bb] = fmaf(-m_use, c, neg_e);
            bscale[bb] = pow2_from_byte(byte);
          }
          if (bb % 4 == 0) sbytes[bb / 4] = 0;
          sbytes[bb / 4] |= byte << (8 * (bb % 4));
        }
        // P~ buffer t&1: its last reader, the product of key tile t-2, completed before S(x, t) was
        // issued (the S issuer waits for it)
        const int pb = t & 1;
        // 32 keys at a time: 16 packed FMAs, 32 ex2, four words of codes, one 16-byte store
        uint8_t* p_row = s.p[x][pb] + r * kPRowBytes;
        uint8_t* d_row = (DBG && dbg) ? p.dbg_codes + static_cast<size_t>(qrow - p.dbg_r0) * (p.Npad / 2) + t * kPRowBytes
                                      : nullptr;
        float tile_sum = 0.f;
#pragma unroll
        for (int cc = 0; cc < kBN / 32; ++cc) {
          float* y = sv + 32 * cc;
          uint4 w4;
          if constexpr (EFQ) {
            // w = sat((2 r + 2) / 7); w times 7 * 2^-149 lands on the subnormal grid, so the product's
            // bit pattern is round(7 w) in [0, 7] (round to nearest even): the code itself
            const float b7 = fmaf(nb[cc], 2.f / 7.f, 2.f / 7.f);
            uint32_t wd[4];
#pragma unroll
            for (int w = 0; w < 4; ++w) {
              float k[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) k[i] = fma_sat(y[8 * w + i], c27, b7);
#pragma unroll
              for (int i = 0; i < 8; i += 2) fmul2_b(k[i], k[i + 1], k[i], k[i + 1], __uint_as_float(7u));
              uint32_t acc = pack_u4x2(0u, __float_as_uint(k[7]), __float_as_uint(k[6]));
              acc = pack_u4x2(acc, __float_as_uint(k[5]), __float_as_uint(k[4]));
              acc = pack_u4x2(acc, __float_as_uint(k[3]), __float_as_uint(k[2]));
              wd[w] = pack_u4x2(acc, __float_as_uint(k[1]), __float_as_uint(k[0]));
            }
            w4 = make_uint4(wd[0], wd[1], wd[2], wd[3]);
          } else {
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
              float x0, x1;
              ffma2_bc(x0, x1, y[i], y[i + 1], c, nb[(32 * cc + i) / kPB]);
              if (PM == 1 && poly_pair<kPolyPairs8>(i / 2)) {
                exp2_codes_poly(y[i], y[i + 1], x0, x1);
              } else {
                y[i] = ex2_approx_ftz(x0);
                y[i + 1] = ex2_approx_ftz(x1);
              }
            }
            w4 = make_uint4(cvt_e2m1x8(y), cvt_e2m1x8(y + 8), cvt_e2m1x8(y + 16), cvt_e2m1x8(y + 24));
          }
          *reinterpret_cast<uint4*>(p_row + ((cc ^ swz) << 4)) = w4;
          if (DBG && dbg) reinterpret_cast<uint4*>(d_row)[cc] = w4;
          if (!PNQ) {   // conventional row sum of the unquantized exponentials
#pragma unroll
            for (int bb = 0; bb < 32 / kPB; ++bb) {
              float b0 = 0.f, b1 = 0.f;
#pragma unroll
              for (int i = 0; i < kPB; i += 2) {
                b0 += y[bb * kPB + i];
                b1 += y[bb * kPB + i + 1];
              }
              tile_sum = fmaf(b0 + b1, bscale[(32 * cc) / kPB + bb], tile_sum);
            }
          }
        }
        if (!PNQ) l = fmaf(alpha, l, tile_sum);
#pragma unroll
        for (int a = 0; a < kNPB / 4; ++a) *reinterpret_cast<uint32_t*>(s.psf[x][pb] + a * 512 + psf_off) = sbytes[a];
        if (DBG && dbg) {
          uint32_t* ds = reinterpret_cast<uint32_t*>(p.dbg_scales + static_cast<size_t>(qrow - p.dbg_r0) *
                                                                        (p.Npad / kPB) + t * kNPB);
#pragma unroll
          for (int a = 0; a < kNPB / 4; ++a) ds[a] = sbytes[a];
        }
        fence_proxy_async_smem();

        // history rescale of O and L (only when some row of this warp saw its max move); O may only
        // be touched once the product of key tile t-1 has landed in it
        if (t > 0 && moved) {
          ok = warp_wait(&s.bar_pv_done[x][pb ^ 1], ((t - 1) >> 1) & 1, abort_flag, p.status, kStatusTimeoutPV | 4);
          if (!ok) break;
          tc_fence_after();
          {
            // O and (PNQ) L in one batch of loads behind one wait, then one batch of stores
            uint32_t raw[D];
#pragma unroll
            for (int cc = 0; cc < D / 32; ++cc)
              tmem_ld32(o_col + cc * 32, *reinterpret_cast<uint32_t(*)[32]>(raw + 32 * cc));
            const uint32_t lv = PNQ ? tmem_ld1(l_col) : 0u;
            tc_wait_ld();
#pragma unroll
            for (int i = 0; i < D; i += 2) {
              float o0, o1;
              fmul2_b(o0, o1, __uint_as_float(raw[i]), __uint_as_float(raw[i + 1]), alpha);
              raw[i] = __float_as_uint(o0);
              raw[i + 1] = __float_as_uint(o1);
            }
#pragma unroll
            for (int cc = 0; cc < D / 32; ++cc)
              tmem_st32(o_col + cc * 32, *reinterpret_cast<const uint32_t(*)[32]>(raw + 32 * cc));
            if (PNQ) tmem_st1(l_col, __float_as_uint(__uint_as_float(lv) * alpha));
          }
          tc_wait_st();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.bar_p_full[x][pb]);
        m = m_new;
      }

      // ---- epilogue: out = O / l (PV products complete in order: the last one covers all)
      if (ok) {
        ok = warp_wait(&s.bar_pv_done[x][(n_kv - 1) & 1], ((n_kv - 1) >> 1) & 1, abort_flag, p.status,
                       kStatusTimeoutPV | 1);
      }
      if (ok) {
        tc_fence_after();
        if (PNQ) {
          l = __uint_as_float(tmem_ld1(l_col));
          tc_wait_ld();
        }
        const float inv_l = 1.f / l;
        // The normalised rows leave through shared memory so that the global writes are whole lines:
        // each warp stages a 32-row x 128-byte chunk (32 fp32 or 64 bf16 columns, its threads' rows)
        // in its quarter of its query tile's P~ buffers, which no product reads any more once the
        // last P~V product has completed, then reads it back four rows per instruction (eight
        // lanes per 128-byte line). 128-byte swizzle: the 16-byte piece j of row r sits at position
        // j ^ (r & 7), so that neither the row-wise writes nor the line-wise reads conflict on banks.
        uint8_t* stage = s.p[x][0] + quarter * 4096;
        const uint32_t row_addr = smem_u32(stage) + static_cast<uint32_t>(lane) * 128u;
        const uint32_t sw = static_cast<uint32_t>(lane) & 7u;
        const int y0 = qt * kBM + quarter * 32;
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t raw[32];
          tmem_ld32(o_col + cc * 32, raw);
          tc_wait_ld();
          const bool half2 = p.out_bf16 && (cc & 1);        // bf16: second half of a 128-byte row
          if (p.out_bf16) {
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint32_t wv[4];
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(raw[v * 8 + 2 * u]) * inv_l,
                                                                __uint_as_float(raw[v * 8 + 2 * u + 1]) * inv_l);
                wv[u] = *reinterpret_cast<const uint32_t*>(&h2);
              }
              st_shared_v4(row_addr + ((((half2 ? 4u : 0u) + v) ^ sw) << 4), wv[0], wv[1], wv[2], wv[3]);
            }
          } else {
#pragma unroll
            for (int v = 0; v < 8; ++v)
              st_shared_v4(row_addr + ((static_cast<uint32_t>(v) ^ sw) << 4),
                           __float_as_uint(__uint_as_float(raw[4 * v]) * inv_l),
                           __float_as_uint(__uint_as_float(raw[4 * v + 1]) * inv_l),
                           __float_as_uint(__uint_as_float(raw[4 * v + 2]) * inv_l),
                           __float_as_uint(__uint_as_float(raw[4 * v + 3]) * inv_l));
          }
          if (!p.out_bf16 || half2) {
            __syncwarp();
            const int es = p.out_bf16 ? 2 : 4;
            const int pc = lane & 7;
            uint8_t* gbase = static_cast<uint8_t*>(p.out) + static_cast<size_t>(bh_q) * p.N * D * es +
                             (p.out_bf16 ? (cc >> 1) * 128 : cc * 128) + pc * 16;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const int rr = 4 * k + (lane >> 3);
              const uint4 val = ld_shared_v4(smem_u32(stage) + rr * 128 + ((pc ^ (rr & 7)) << 4));
              if (y0 + rr < p.N) *reinterpret_cast<uint4*>(gbase + static_cast<size_t>(y0 + rr) * D * es) = val;
            }
            __syncwarp();     // the stage is read before the next chunk overwrites it
          }
        }
      }
      tc_fence_before();
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, int PM, bool DBG, bool NV, int WS>
static cudaError_t launch_k(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                            const AttnParams& p, cudaStream_t stream) {
  const size_t smem = smem_bytes<D>();
  // the softmax warpgroups' register increase is served from the block's launch allocation: a
  // build with fewer registers per thread than the split assumes would make it wait forever
  static int regs = -1;
  if (regs < 0) {
    cudaFuncAttributes fa;
    cudaError_t ea = cudaFuncGetAttributes(&fa, mxattn_fwd_kernel<D, PM, DBG, NV, WS>);
    if (ea != cudaSuccess) return ea;
    regs = fa.numRegs;
  }
  if (regs != Layout<WS>::kLaunchRegs) return cudaErrorInvalidConfiguration;
  cudaError_t e = cudaFuncSetAttribute(mxattn_fwd_kernel<D, PM, DBG, NV, WS>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const unsigned n_units = static_cast<unsigned>((p.Npad / kBM + 1) / 2);
  const unsigned grid = static_cast<unsigned>(p.B) * p.Hq * n_units;
  mxattn_fwd_kernel<D, PM, DBG, NV, WS><<<grid, Layout<WS>::kThreads, smem, stream>>>(tmQ, tmK, tmV, p);
  return cudaGetLastError();
}

// Softmax layout per launch (measured on the benchmark workloads): two threads per row for
// exp-then-quantize without a causal mask (video-DiT PNQ +2%, NVFP4 +2%, pnq = 0 +1%); one thread
// per row for the exp-free rule (the two-thread layout is 8% slower there) and for causal
// attention (1% slower there: more of its time is per-unit work).
template <int D, int PM, bool DBG, bool NV>
static cudaError_t launch_w(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                            const AttnParams& p, cudaStream_t stream) {
  if (PM != 2 && !p.causal) return launch_k<D, PM, DBG, NV, 8>(tmQ, tmK, tmV, p, stream);
  return launch_k<D, PM, DBG, NV, 4>(tmQ, tmK, tmV, p, stream);
}

template <int D, bool NV>
static cudaError_t launch_f(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                            const AttnParams& p, cudaStream_t stream) {
  const bool dbg = p.dbg_codes != nullptr;
  if (p.pnq == 2) {
    if constexpr (NV) return cudaErrorInvalidValue;    // the exp-free rule is MXFP4 only
    else return dbg ? launch_w<D, 2, true, NV>(tmQ, tmK, tmV, p, stream)
                    : launch_w<D, 2, false, NV>(tmQ, tmK, tmV, p, stream);
  }
  if (p.pnq == 1) return dbg ? launch_w<D, 1, true, NV>(tmQ, tmK, tmV, p, stream)
                             : launch_w<D, 1, false, NV>(tmQ, tmK, tmV, p, stream);
  return dbg ? launch_w<D, 0, true, NV>(tmQ, tmK, tmV, p, stream)
             : launch_w<D, 0, false, NV>(tmQ, tmK, tmV, p, stream);
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

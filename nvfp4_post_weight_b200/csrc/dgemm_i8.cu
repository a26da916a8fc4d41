// fp64-accurate GEMM on the 5th-generation tensor cores through int8 slices:
//   C = beta C + alpha P Q^T   (P: M x K, Q: N x K row-major fp64, C: M x N)
// with the options of dgemm_nt (batch, lower tiles, triangular P, C2 = C^T).
//
// tcgen05 has no fp64 kind, but its int8 kind multiplies exactly into int32.
// Each row of P (and of Q) is scaled by a power of two so that its largest
// entry lies in [1/4, 1/2), and the scaled values are cut into S signed 7-bit
// slices:  x = sum_t a_t 2^(-7 (t + 1)) + r,  a_t in [-64, 64] (balanced
// base-128 digits of x rounded to a multiple of 2^(-7 S)), |r| <= 2^(-7 S - 1)
// (the splitting of Ozaki et al., "Error-free
// transformations of matrix multiplication by using fast routines of matrix
// multiplication and its applications", Numer. Algorithms 59 (2012), with
// integer slices).  Then
//   (P Q^T)_mn = 2^(e_m + e_n) sum_{t,u} 2^(-7 (t + u + 2)) (A_t B_u^T)_mn,
// every slice product is exact in int32, and the products of one level
// l = t + u share an int32 TMEM accumulator (exact: |sum| < 2^31 for K < 2^16).
// Levels l > S - 1 are dropped: together with the digits' rounding they weigh
// less than 2^(-7 S + 3) of the row and column maxima, 2^-39 for S = 6.  The
// factorisation's result U is stored in fp32 (relative rounding 2^-24), and
// even amplified by the damped Hessian's condition number (1.6e4 on the
// hardest workload measured) this error stays at or below that rounding.
// The levels are combined in fp64 in the epilogue.
//
// Persistent kernel, one CTA per SM, 128 x 64 output tiles:
//   warp 0     TMA producer: a 2-stage ring, each stage 64 K-bytes of all S
//              slices of A (128 rows) and B (64 rows), one 3-D load per
//              operand (SWIZZLE_64B: two MMAs' K per 64-byte row; rows of
//              32 bytes took twice the TMA requests per byte and ran 6-8%
//              slower even with a deeper ring)
//   warp 1     MMA issuer.  The B slices of a stage lie one after another and
//              so do the S level accumulators in TMEM (64 columns each), so
//              A_t times the stacked B_0 .. B_{S-1-t} adds A_t B_u^T to level
//              t + u for all u in one MMA of N = 64 (S - t) (cut at 256): 8
//              MMAs per 32-byte K step instead of S (S + 1) / 2 = 21 narrow
//              ones
//   warps 2-5  epilogue: levels summed in fp64 straight out of TMEM, TMEM
//              handed back (the next tile's MMAs start), then the tile is
//              scaled by the row and column exponents and written through a
//              shared-memory staging tile (C coalesced by rows, C2 = C^T by
//              columns) while the tensor cores work on the next tile.
// Tiles are ordered so that the work per tile never grows along the order
// (triangular P: longest K ranges first) and dealt to the CTAs in rounds,
// every other round backwards.  Every wait is bounded; a wait that runs out
// records NVFP4_ERR_TIMEOUT and the CTA drains its copies and MMAs and frees
// TMEM before it returns.
#include <cuda.h>

#include "common.cuh"
#include "sm100.cuh"

namespace nvfp4 {
namespace {

using namespace sm100;

constexpr int S = 6;                     // slices per value
constexpr int IM = 128, IN = 64;         // output tile
constexpr int KC = 64;                   // K bytes (int8 values) per stage: two MMAs' K
constexpr int kIStages = 2;
constexpr uint32_t kASlice = IM * KC;    // 4 KB
constexpr uint32_t kBSlice = IN * KC;    // 2 KB
constexpr uint32_t kIStage = S * (kASlice + kBSlice);   // 36 KB
constexpr int kIThreads = 192;
constexpr uint32_t kITmemCols = 512;     // S levels x IN columns = 448
constexpr int kTilePitch = IN + 1;       // staged fp64 result tile, IM x kTilePitch
constexpr size_t kITileBytes = sizeof(double) * IM * kTilePitch;
constexpr size_t kISmem = kIStages * kIStage + kITileBytes + 1024 + 256;

struct IBars {
  uint64_t full[kIStages], empty[kIStages], acc_full, acc_empty, done;
  uint32_t tmem;
  int abort;
};

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// K-major operand in the canonical 64-byte-swizzled layout: rows of 64 bytes
// (two MMAs' K; the second MMA's operand starts 32 bytes into the row),
// 8-row groups 512 bytes apart.
__device__ __forceinline__ uint64_t desc_sw64(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFF);
  d |= (uint64_t)1 << 16;             // leading byte offset (unused when K fits a row)
  d |= (uint64_t)(512 >> 4) << 32;    // stride byte offset: 8 rows x 64 B
  d |= (uint64_t)1 << 46;             // descriptor version (sm_100)
  d |= (uint64_t)4 << 61;             // SWIZZLE_64B
  return d;
}

// AND of v over the 128 threads that take named barrier `id` (a barrier too).
__device__ __forceinline__ bool bar_and_128(int id, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void mma_i8(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 64 consecutive 32-bit columns of this thread's TMEM lane (warp-wide), one
// load and its wait in one statement.
__device__ __forceinline__ void tmem_ld64_raw(uint32_t taddr, uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(taddr)
      : "memory");
}

// The int32 v as a double, exactly, on the integer and fp64 pipes instead of
// the slower conversion unit: the double with high word 0x43300000 and low
// word v + 2^31 (as unsigned) is 2^52 + 2^31 + v, an integer below 2^53, and
// subtracting 2^52 + 2^31 leaves v without rounding.
__device__ __forceinline__ double i32_to_f64(uint32_t v) {
  return __dsub_rn(__hiloint2double(0x43300000, (int)(v ^ 0x80000000u)),
                   4503601774854144.0 /* 2^52 + 2^31 */);
}

// D = s32, A and B signed 8-bit, both K-major, M = 128, N = n (a multiple of
// 16 up to kMaxN).
constexpr int kMaxN = 256;
__host__ __device__ constexpr uint32_t idesc_i8(int n) {
  return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) |
         ((uint32_t)(IM >> 4) << 24);
}

// Slices of one fp64 matrix (rows x K, leading dimension ld, batch entries
// `stride` apart): slice t of row r (batch b) at out + t * plane +
// (b * rows + r) * kp, exponent at e[b * rows + r].  One CTA per row (blockIdx.x
// = r, blockIdx.y = b), eight consecutive values per thread and chunk; the
// first chunk stays in registers between the max pass and the digit pass.
//
// Each scaled value v = 2^(7 S) 2^-ex x (|v| < 2^(7 S - 1)) is rounded once to an
// integer, ties to even, by adding 1.5 * 2^52: the sum's 52-bit fraction is
// then f = 2^51 + v, whose low 28 bits are those of v and whose bits from 28
// up, less 2^23, are floor(v / 2^28).  The balanced base-128 digits are cut
// from the bottom with 32-bit steps: four from the low 28 bits (whose carry,
// 0 or 1, goes to the high part), S - 5 from the high part, and the rest is
// the top digit.  Digit t in [-64, 63] for t > 0, the top one in [-64, 64].
__device__ __forceinline__ void load8(const double* __restrict__ x, int64_t k, int64_t K,
                                      double (&xv)[8]) {
  if (k + 8 <= K && ((reinterpret_cast<uintptr_t>(x + k) & 15) == 0)) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const double2 p2 = reinterpret_cast<const double2*>(x + k)[q];
      xv[2 * q] = p2.x;
      xv[2 * q + 1] = p2.y;
    }
  } else {
#pragma unroll
    for (int q = 0; q < 8; ++q) xv[q] = k + q < K ? x[k + q] : 0.0;
  }
}

__device__ __forceinline__ void digits8(const double (&xv)[8], double to_int, int8_t* o,
                                        int64_t plane) {
  // |v| < 2^(7 S - 1) must stay below 2^51 for the rounding by addition
  static_assert(S >= 6 && S <= 7, "four low digits, S - 5 high ones and the top digit");
  uint32_t w[S][2];
#pragma unroll
  for (int t = 0; t < S; ++t) w[t][0] = w[t][1] = 0u;
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const double tq = __dadd_rn(__dmul_rn(xv[q], to_int), 0x1.8p52);
    const uint32_t lw = (uint32_t)__double2loint(tq), hw = (uint32_t)__double2hiint(tq);
    int lo = (int)(lw & 0x0FFFFFFFu);
    int hi = (int)(((hw & 0xFFFFFu) << 4) | (lw >> 28)) - (1 << 23);
    const int sh = 8 * (q & 3);
#pragma unroll
    for (int t = S - 1; t >= S - 4; --t) {
      const int a = ((lo + 64) & 127) - 64;
      lo = (lo - a) >> 7;
      w[t][q >> 2] |= ((uint32_t)a & 0xFFu) << sh;
    }
    hi += lo;
#pragma unroll
    for (int t = S - 5; t >= 1; --t) {
      const int a = ((hi + 64) & 127) - 64;
      hi = (hi - a) >> 7;
      w[t][q >> 2] |= ((uint32_t)a & 0xFFu) << sh;
    }
    w[0][q >> 2] |= ((uint32_t)hi & 0xFFu) << sh;
  }
#pragma unroll
  for (int t = 0; t < S; ++t) *reinterpret_cast<uint2*>(o + t * plane) = make_uint2(w[t][0], w[t][1]);
}

__global__ void __launch_bounds__(256) slice_rows_kernel(const double* __restrict__ X,
                                                         int64_t rows, int64_t K, int64_t ld,
                                                         int64_t stride, int64_t kp,
                                                         int64_t plane,
                                                         int8_t* __restrict__ out,
                                                         int* __restrict__ e) {
  __shared__ double wmax[8];
  pdl_wait();
  const int64_t r = blockIdx.x;
  const int b = blockIdx.y;
  const int tid = threadIdx.x, T = blockDim.x, lane = tid & 31;
  const double* x = X + b * stride + r * ld;
  const int64_t k0 = 8 * tid, step = 8 * (int64_t)T;
  double xv[8];
  load8(x, k0, K, xv);   // (zeros past K: kp and K are multiples of 16)
  double m = 0.0;
#pragma unroll
  for (int q = 0; q < 8; ++q) m = fmax(m, fabs(xv[q]));
  for (int64_t k = k0 + step; k < kp; k += step) {
    double yv[8];
    load8(x, k, K, yv);
#pragma unroll
    for (int q = 0; q < 8; ++q) m = fmax(m, fabs(yv[q]));
  }
  for (int o = 16; o > 0; o >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) wmax[tid >> 5] = m;
  __syncthreads();
  m = 0.0;
  for (int w = 0; w < (T >> 5); ++w) m = fmax(m, wmax[w]);
  // 2^-ex m in [1/4, 1/2): the first slice rint(128 x) stays within [-64, 64]
  const int ex = m > 0.0 ? ilogb(m) + 2 : 0;
  const double to_int = scalbn(1.0, 7 * S - ex);   // exact power of two
  const int64_t row = b * rows + r;
  if (tid == 0) e[row] = ex;
  int8_t* o = out + row * kp;
  if (k0 < kp) digits8(xv, to_int, o + k0, plane);
  for (int64_t k = k0 + step; k < kp; k += step) {
    double yv[8];
    load8(x, k, K, yv);
    digits8(yv, to_int, o + k, plane);
  }
}

// Output tiles of one launch.  A lower result (all K ranges equal) takes, per
// batch entry, the tiles that reach the diagonal or below it (n0 <= m0 + 127:
// row tm holds min(2 tm + 2, nt) of them and starts at tm (tm + 1)).  A full
// result is ordered by tile row first, then batch entry and column, with the
// rows of a triangular P in the order of falling K range (ktri 1: ascending,
// ktri 2: descending), so that the work per tile never grows along the order;
// where the B slices are far larger than L2, by groups of tile rows (below).
constexpr int kGroupRows = 16;
struct ITiles {
  int mt, nt, batch, lower, ktri, grouped;
  __device__ int per() const {
    if (!lower) return mt * nt;
    return mt * (mt + 1) - (nt < 2 * mt ? 2 * mt - nt : 0);   // the last row may be short
  }
  __device__ int count() const { return per() * batch; }
  __device__ void get(int t, int& tm, int& tn, int& b) const {
    if (lower) {
      const int p = per();
      b = t / p;
      t -= b * p;
      int r = (int)((sqrtf(4.f * (float)t + 1.f) - 1.f) * 0.5f);
      while ((r + 1) * (r + 2) <= t) ++r;
      while (r * (r + 1) > t) --r;
      tm = r;
      tn = t - r * (r + 1);
    } else if (!grouped) {
      const int row = nt * batch;
      const int i = t / row;
      t -= i * row;
      b = t / nt;
      tn = t - b * nt;
      tm = ktri == 2 ? mt - 1 - i : i;
    } else {
      // B slices far beyond L2: groups of kGroupRows tile rows, inside a group
      // batch entry by batch entry and column by column, so that the CTAs of
      // a round share a few A row slabs and a short run of B column slabs in
      // L2 (row-major order would stream every B slab from DRAM once per
      // round); the groups keep the falling K-range order
      const int pg = kGroupRows * nt * batch;
      const int g = t / pg;
      t -= g * pg;
      const int r = (mt - g * kGroupRows) < kGroupRows ? (mt - g * kGroupRows) : kGroupRows;
      b = t / (r * nt);
      t -= b * r * nt;
      tn = t / r;
      const int i = g * kGroupRows + t % r;
      tm = ktri == 2 ? mt - 1 - i : i;
    }
  }
  // The k-th tile of CTA c among g: rounds of g tiles, every other round
  // walked backwards, so that a CTA given a heavy tile in one round gets a
  // light one in the next.
  __device__ static int pick(int k, int c, int g) { return k * g + ((k & 1) ? g - 1 - c : c); }
};

__global__ void __launch_bounds__(kIThreads, 1)
    dgemm_i8_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const int* __restrict__ eA, const int* __restrict__ eB, int M, int N, int K,
                    double alpha, double beta, double* __restrict__ C, int64_t ldc,
                    int64_t strideC, double* __restrict__ C2, int64_t ldc2, int64_t strideC2,
                    ITiles ts, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  double* tile = reinterpret_cast<double*>(ring + kIStages * kIStage);
  IBars* sm = reinterpret_cast<IBars*>(ring + kIStages * kIStage + kITileBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = ts.count();
  auto k_range = [&](int tm, int& kc0, int& nk) {
    const int m0 = tm * IM;
    int kbeg = 0, kend = K;
    if (ts.ktri == 1) kbeg = (m0 / KC) * KC;
    if (ts.ktri == 2) kend = (m0 + IM) < K ? (m0 + IM) : K;
    kc0 = kbeg / KC;
    nk = kend > kbeg ? (kend - kbeg + KC - 1) / KC : 0;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kIStages; ++s) {
      mbar_init(&sm->full[s], 1);
      mbar_init(&sm->empty[s], 1);
    }
    mbar_init(&sm->acc_full, 1);
    mbar_init(&sm->acc_empty, 128);
    mbar_init(&sm->done, 1);
    sm->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&sm->tmem, kITmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm->tmem;
  pdl_wait();

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer
    tma_prefetch(&tmA);
    tma_prefetch(&tmB);
    int g = 0;   // stages issued over all tiles
    bool ok = true;
    for (int k = 0; ok && k * (int)gridDim.x < n_tiles; ++k) {
      const int t = ITiles::pick(k, blockIdx.x, gridDim.x);
      if (t >= n_tiles) continue;
      int tm, tn, bz, kc0, nk;
      ts.get(t, tm, tn, bz);
      k_range(tm, kc0, nk);
#ifdef NVFP4_DEBUG
      if (!NVFP4_DCHECK(bz >= 0 && bz < ts.batch && tm >= 0 && tm < ts.mt && tn >= 0 &&
                            tn < ts.nt && (!ts.lower || tn * IN <= tm * IM + IM - 1),
                        status))
        continue;   // debug build: a tile outside the output is skipped by every role
#endif
      for (int i = 0; i < nk; ++i, ++g) {
        const int s = g % kIStages;
        if ((g >= kIStages && !mbar_wait(&sm->empty[s], ((g / kIStages) - 1) & 1)) ||
            *reinterpret_cast<volatile int*>(&sm->abort)) {
          atomicExch(&sm->abort, 1);
          atomicCAS(status, 0, (int)NVFP4_ERR_TIMEOUT);
          ok = false;
          break;
        }
        uint8_t* st = ring + s * kIStage;
        mbar_arrive_expect_tx(&sm->full[s], kIStage);
        tma_load_3d(st, &tmA, &sm->full[s], (kc0 + i) * KC, bz * M + tm * IM, 0);
        tma_load_3d(st + S * kASlice, &tmB, &sm->full[s], (kc0 + i) * KC, bz * N + tn * IN, 0);
      }
    }
    for (int i = g - kIStages < 0 ? 0 : g - kIStages; i < g; ++i)
      mbar_wait_drain(&sm->full[i % kIStages], (i / kIStages) & 1);
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    int g = 0, lt = 0;
    bool ok = true;
    for (int k = 0; ok && k * (int)gridDim.x < n_tiles; ++k) {
      const int t = ITiles::pick(k, blockIdx.x, gridDim.x);
      if (t >= n_tiles) continue;
      int tm, tn, bz, kc0, nk;
      ts.get(t, tm, tn, bz);
      k_range(tm, kc0, nk);
#ifdef NVFP4_DEBUG
      if (!NVFP4_DCHECK(bz >= 0 && bz < ts.batch && tm >= 0 && tm < ts.mt && tn >= 0 &&
                            tn < ts.nt && (!ts.lower || tn * IN <= tm * IM + IM - 1),
                        status))
        continue;   // debug build: a tile outside the output is skipped by every role
#endif
      // the epilogue has read the previous tile's accumulators out of TMEM
      if (lt > 0 && !mbar_wait(&sm->acc_empty, (lt - 1) & 1)) {
        atomicExch(&sm->abort, 1);
        atomicCAS(status, 0, (int)NVFP4_ERR_TIMEOUT);
        break;
      }
      tc_fence_after();
      for (int i = 0; i < nk; ++i, ++g) {
        const int s = g % kIStages;
        if (!mbar_wait(&sm->full[s], (g / kIStages) & 1)) {
          atomicExch(&sm->abort, 1);
          atomicCAS(status, 0, (int)NVFP4_ERR_TIMEOUT);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a0 = smem_u32(ring + s * kIStage), b0 = a0 + S * kASlice;
        // A_t times the stacked B_0 .. B_{S-1-t} (N = IN (S - t), cut at
        // 256) adds A_t B_u^T to level t + u for every u at once: the B
        // slices lie one after another in the stage and so do the level
        // accumulators in TMEM
#pragma unroll
        for (int kk = 0; kk < KC / 32; ++kk)
#pragma unroll
        for (int t = 0; t < S; ++t)
#pragma unroll
          for (int c0 = 0; c0 < IN * (S - t); c0 += kMaxN)
            mma_i8(tmem + IN * t + c0, desc_sw64(a0 + t * kASlice + 32 * kk),
                   desc_sw64(b0 + c0 * KC + 32 * kk),
                   idesc_i8(IN * (S - t) - c0 < kMaxN ? IN * (S - t) - c0 : kMaxN),
                   (i > 0 || t > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&sm->empty[s]);
      }
      mma_commit(&sm->acc_full);   // arrives when this tile's MMAs are done (also if nk == 0)
      ++lt;
    }
    // nothing of this thread's may still run on the tensor cores when TMEM is
    // freed, also after a wait ran out
    mma_commit(&sm->done);
    mbar_wait_drain(&sm->done, 0);
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue
    // (1) the levels of each row are summed in fp64 straight out of TMEM,
    // scaled by 2^(e_m - 14) and staged in shared memory, and TMEM is handed
    // back to the MMA warp (the next tile's products start); (2) the four
    // warps write C row by row and C2 column by column, both coalesced, with
    // the column factors 2^(e_n).
    const int q = warp & 3;
    const int r = q * 32 + lane;   // tile row = TMEM lane
    int lt = 0;
    for (int k = 0; k * (int)gridDim.x < n_tiles; ++k) {
      const int t = ITiles::pick(k, blockIdx.x, gridDim.x);
      if (t >= n_tiles) continue;
      int tm, tn, bz, kc0, nk;
      ts.get(t, tm, tn, bz);
      k_range(tm, kc0, nk);
#ifdef NVFP4_DEBUG
      if (!NVFP4_DCHECK(bz >= 0 && bz < ts.batch && tm >= 0 && tm < ts.mt && tn >= 0 &&
                            tn < ts.nt && (!ts.lower || tn * IN <= tm * IM + IM - 1),
                        status))
        continue;   // debug build: a tile outside the output is skipped by every role
#endif
      const int m0 = tm * IM, n0 = tn * IN;
      const bool mine = __all_sync(0xffffffffu, mbar_wait(&sm->acc_full, lt & 1));
      tc_fence_after();
      double acc[IN];
#pragma unroll
      for (int j = 0; j < IN; ++j) acc[j] = 0.0;
      if (mine && nk > 0) {
        // levels from the smallest weight up: acc = sum_l 2^(-7 l) v_l
#pragma unroll 1
        for (int l = S - 1; l >= 0; --l) {
          uint32_t v[IN];
          tmem_ld64_raw(tmem + ((uint32_t)(q * 32) << 16) + l * IN, v);
#pragma unroll
          for (int j = 0; j < IN; ++j)
            acc[j] = fma(acc[j], 0.0078125 /* 2^-7 */, i32_to_f64(v[j]));
        }
      }
      tc_fence_before();
      if (mine) mbar_arrive(&sm->acc_empty);
      // one decision for the four warps; the barrier also keeps the staged
      // tile from being overwritten before the previous tile's C writes
      if (!bar_and_128(1, mine && !*reinterpret_cast<volatile int*>(&sm->abort))) {
        if (threadIdx.x == 64) atomicCAS(status, 0, (int)NVFP4_ERR_TIMEOUT);
        break;
      }
      const int m = m0 + r;
      const double fm = m < M ? scalbn(alpha, eA[bz * M + m] - 14) : 0.0;   // level 0 weighs 2^-14
#pragma unroll
      for (int j = 0; j < IN; ++j) tile[r * kTilePitch + j] = acc[j] * fm;
      asm volatile("bar.sync 1, 128;" ::: "memory");
      double fn[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int n = n0 + lane + 32 * h;
        fn[h] = n < N ? scalbn(1.0, eB[bz * N + n]) : 0.0;
      }
      double* __restrict__ Cb = C + bz * strideC;
      // the warp's 32 rows: all their C loads are issued before any store
      double old[IM / 4][2];
#pragma unroll
      for (int i = 0; i < IM / 4; ++i) {
        const int mm = m0 + q + 4 * i;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int n = n0 + lane + 32 * h;
          old[i][h] = (beta != 0.0 && mm < M && n < N) ? Cb[(int64_t)mm * ldc + n] : 0.0;
        }
      }
#pragma unroll
      for (int i = 0; i < IM / 4; ++i) {
        const int mm = m0 + q + 4 * i;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int n = n0 + lane + 32 * h;
          if (mm < M && n < N) {
            double xv = tile[(q + 4 * i) * kTilePitch + lane + 32 * h] * fn[h];
            if (beta != 0.0) xv = fma(beta, old[i][h], xv);
            Cb[(int64_t)mm * ldc + n] = xv;
          }
        }
      }
      if (C2) {
        double* C2b = C2 + bz * strideC2;
        for (int j = q; j < IN; j += 4) {
          const int n = n0 + j;
          if (n >= N) break;
          const double f = scalbn(1.0, eB[bz * N + n]);
#pragma unroll
          for (int h = 0; h < IM / 32; ++h) {
            const int mm = m0 + lane + 32 * h;
            if (mm < M) C2b[(int64_t)n * ldc2 + mm] = tile[(lane + 32 * h) * kTilePitch + j] * f;
          }
        }
      }
      ++lt;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kITmemCols);
  }
}

// 3-D map of the slices: (K bytes, batch * rows, S), box {32, box_rows, S}.
bool encode_slices(CUtensorMap* map, const int8_t* base, int64_t K, int64_t total_rows,
                   int64_t kp, int64_t plane, int box_rows) {
  const uint64_t dims[3] = {(uint64_t)K, (uint64_t)total_rows, (uint64_t)S};
  const uint64_t strides[2] = {(uint64_t)kp, (uint64_t)plane};
  const uint32_t box[3] = {(uint32_t)KC, (uint32_t)box_rows, (uint32_t)S};
  return encode_tmap_nd(map, base, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, dims, strides, box,
                        CU_TENSOR_MAP_SWIZZLE_64B);
}

nvfp4_status slice(const double* X, int64_t rows, int64_t K, int64_t ld, int64_t stride,
                   int batch, int8_t* out, int* e, int64_t kp, int64_t plane, cudaStream_t st) {
  // one CTA per row, one 8-value chunk per thread up to K = 2048
  int threads = (int)((kp / 8 + 31) / 32 * 32);
  threads = threads < 32 ? 32 : (threads > 256 ? 256 : threads);
  const dim3 grid((unsigned)rows, (unsigned)batch);
  NVFP4_CUDA_TRY(launch_chained(slice_rows_kernel, grid, dim3(threads), 0, st, X, rows, K, ld,
                                stride, kp, plane, out, e));
  count_launches(1);
  return NVFP4_OK;
}

}  // namespace

size_t dgemm_i8_scratch_bytes(int64_t M, int64_t N, int64_t K, int batch) {
  const int64_t kp = (K + 63) / 64 * 64;
  return align256((size_t)S * batch * M * kp) + align256((size_t)S * batch * N * kp) +
         align256(sizeof(int) * batch * (M + N));
}

nvfp4_status dgemm_i8(int M, int N, int K, double alpha, const double* P, int64_t ldp,
                      int64_t strideP, const double* Q, int64_t ldq, int64_t strideQ,
                      double beta, double* C, int64_t ldc, int64_t strideC, double* C2,
                      int64_t ldc2, int64_t strideC2, int batch, int lower, int ktri,
                      void* scratch, size_t scratch_bytes, int* status, cudaStream_t st) {
  if (M <= 0 || N <= 0 || batch <= 0) return NVFP4_OK;
  // K < 2^16 keeps a level's int32 sum exact: S pairs x K x 64 x 64 < 2^31
  if ((C2 && beta != 0.0) || (lower && M != N) || ktri < 0 || ktri > 2 || !status || K <= 0 ||
      K >= (1 << 16) || (K % 16) != 0 || batch > 65535)
    return NVFP4_ERR_INVALID_ARG;
  if (scratch_bytes < dgemm_i8_scratch_bytes(M, N, K, batch)) return NVFP4_ERR_WORKSPACE;
  ProfileScope ps(kPhaseFactorI8, st);
  {
    double f = 2.0 * M * N * K;
    if (lower) f = 2.0 * ((double)N * (N + 1) / 2) * K;
    if (ktri != 0 && M <= K)
      f = 2.0 * N * ((double)M * (M + 1) / 2 + (double)M * (K - M) * (ktri == 1));
    add_phase_work(f * batch);
  }
  const int64_t kp = (K + 63) / 64 * 64;
  const int64_t planeA = (int64_t)batch * M * kp, planeB = (int64_t)batch * N * kp;
  char* p = static_cast<char*>(scratch);
  int8_t* A = reinterpret_cast<int8_t*>(p);
  p += align256((size_t)S * planeA);
  int8_t* Bs = reinterpret_cast<int8_t*>(p);
  p += align256((size_t)S * planeB);
  int* eA = reinterpret_cast<int*>(p);
  int* eB = eA + (int64_t)batch * M;
  // P and Q are the same matrix in a symmetric update: slice it once
  const bool same = (P == Q && ldp == ldq && strideP == strideQ && M == N);
  nvfp4_status s = slice(P, M, K, ldp, strideP, batch, A, eA, kp, planeA, st);
  if (s != NVFP4_OK) return s;
  const int8_t* Bsrc = same ? A : Bs;
  const int* eBsrc = same ? eA : eB;
  if (!same) {
    s = slice(Q, N, K, ldq, strideQ, batch, Bs, eB, kp, planeB, st);
    if (s != NVFP4_OK) return s;
  }
  CUtensorMap ma, mb;
  if (!encode_slices(&ma, A, K, (int64_t)batch * M, kp, planeA, IM) ||
      !encode_slices(&mb, Bsrc, K, (int64_t)batch * N, kp, same ? planeA : planeB, IN))
    return NVFP4_ERR_CUDA;
  // B slices past 256 MB (twice L2): group the tile rows
  const int grouped = !lower && (int64_t)S * batch * N * kp > (int64_t(256) << 20);
  const ITiles ts{(M + IM - 1) / IM, (N + IN - 1) / IN, batch, lower, ktri, grouped};
  const int64_t n_tiles =
      (int64_t)(lower ? (int64_t)ts.mt * (ts.mt + 1) : (int64_t)ts.mt * ts.nt) * batch;
  if (n_tiles > (1ll << 30)) return NVFP4_ERR_SHAPE;
  const int sms = num_sms();
  const dim3 grid((unsigned)(n_tiles < sms ? n_tiles : sms));
  NVFP4_CUDA_TRY(cudaFuncSetAttribute(dgemm_i8_kernel,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kISmem));
  NVFP4_CUDA_TRY(launch_chained(dgemm_i8_kernel, grid, dim3(kIThreads), kISmem, st, ma, mb, eA,
                                eBsrc, M, N, K, alpha, beta, C, ldc, strideC, C2, ldc2, strideC2,
                                ts, status));
  count_launches(1);
  return NVFP4_OK;
}

}  // namespace nvfp4

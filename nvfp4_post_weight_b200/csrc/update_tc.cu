// a8 on the tensor cores: the lazy-batch trailing update
//   W~[:, e:] -= Delta U[c0:c0+128, e:]
// "Replay the Curvature" (arXiv 2609.36654v1), Abstract: in GPTQ every
// quantized column updates the columns after it; lazy batching applies a whole
// batch of 128 columns' updates at once, which is a GEMM with K = 128.
//
// Precision: W~ stays fp64 (the replay decisions need it); the product is
// taken as 3xTF32 on tcgen05 (kind::tf32): Delta = Dh + Dl and U = Uh + Ul
// with Dh, Uh rounded to tf32, and Delta U ~ Dh Uh + Dh Ul + Dl Uh.  The
// tensor cores' fp32 accumulation drops low bits at every step, so the main
// term Dh Uh is split over two TMEM accumulators of K = 64 each (8 steps), the
// two small cross terms share a third; the epilogue adds the three in fp64
// and subtracts the sum from W~.
//
// Both operands are K-major (Uh/Ul hold the batch's rows of U transposed,
// 128 K values per column), in the canonical 128-byte-swizzled layout.
//
// The kernel is bound by the fp64 W~ traffic (read and written once per
// batch), so shared memory goes to keeping that traffic in flight: four
// 32 KB half-tile W~ buffers (two 128 x 64 tiles), loaded by TMA ahead of the
// MMAs that need them and written back by TMA stores; the small operands
// (Dh/Dl, Uh/Ul: L2-resident) stream through a 2-stage ring.
//
// Persistent CTA per SM, warp-specialised, tiles in column-major order (the CTAs
// running at once share a U tile in L2):
//   warp 0     TMA producer: per tile, the two W~ halves first (the long HBM
//              latency), then 4 K-chunks of (Dh, Dl, Uh, Ul)
//   warp 1     MMA issuer, 12 MMAs (M=128, N=64, K=8) per K chunk
//   warps 2-5  epilogue: per half tile, TMEM -> registers, W~ -= sum in the
//              shared-memory buffer (row r's 16-byte chunk j sits at position
//              j ^ (r % 8): the 128-byte swizzle)
//   warp 6     store: writes each finished half back with a TMA store and
//              frees a buffer once its store has read it (one store group is
//              kept in flight, so the epilogue never waits on a store)
#include <cuda.h>

#include "common.cuh"
#include "sm100.cuh"

namespace nvfp4 {
namespace {

using namespace sm100;

constexpr int UM = 128;                        // rows per tile
constexpr int UN = 64;                         // columns per tile
constexpr int UK = kLazyBatch;                 // 128
constexpr int KC = 32;                         // K per chunk (128 B of fp32)
constexpr int kNChunks = UK / KC;              // 4
constexpr uint32_t kAPart = UM * KC * 4;       // 16 KB: Dh or Dl chunk
constexpr uint32_t kBPart = UN * KC * 4;       // 8 KB: Uh or Ul chunk
constexpr uint32_t kStage = 2 * kAPart + 2 * kBPart;   // 48 KB
constexpr int kStages = 2;
constexpr int WBOX = 16;                       // fp64 per TMA box row (128 B)
constexpr uint32_t kWBox = UM * WBOX * 8;      // 16 KB
constexpr uint32_t kWHalf = 2 * kWBox;         // 32 columns = 32 KB
constexpr int kWBufs = 4;                      // half-tile buffers (2 tiles)
constexpr int kThreads = 224;                 // 7 warps
constexpr uint32_t kBufCols = 256;             // TMEM columns between the two accumulators
constexpr uint32_t kTmemCols = 512;
constexpr size_t kSmem = kStages * kStage + kWBufs * kWHalf + 1024 + 256;

struct Smem {
  uint64_t full[kStages], empty[kStages];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t w_full[kWBufs], w_written[kWBufs], w_empty[kWBufs];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ void give_up(Smem* sm, int* status) {
  atomicExch(&sm->abort, 1);
  atomicCAS(status, 0, (int)NVFP4_ERR_TIMEOUT);
}
__device__ __forceinline__ bool aborted(Smem* sm) {
  return *reinterpret_cast<volatile int*>(&sm->abort) != 0;
}

// L2 policies: W~ streams through once per batch (evict first); the small
// operands Dh/Dl and Uh/Ul are re-read by every tile (evict last), and would
// otherwise be pushed out of L2 by the W~ stream.
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// The operands are 3-D: (columns, rows, problem of the group).
__device__ __forceinline__ void tma_load_3d_hint(void* dst, const CUtensorMap* map,
                                                 uint64_t* bar, int c0, int c1, int c2,
                                                 uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(smem_u32(dst)),
      "l"(map), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "l"(policy)
      : "memory");
}

// TMA tile store from shared memory (out-of-range parts are not written).
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int c0,
                                             int c1, int c2, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group.L2::cache_hint"
      " [%0, {%2, %3, %4}], [%1], %5;" ::"l"(map),
      "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2), "l"(policy)
      : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read_all_but_one() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() {    // all committed stores complete
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

__global__ void __launch_bounds__(kThreads, 1)
    update_tc_kernel(const __grid_constant__ CUtensorMap tmDh,
                     const __grid_constant__ CUtensorMap tmDl,
                     const __grid_constant__ CUtensorMap tmUh,
                     const __grid_constant__ CUtensorMap tmUl,
                     const __grid_constant__ CUtensorMap tmW, int e, int n_rb, int n_cols,
                     int n_tiles, int kofs, int nkb, int keep_w, int* status) {
  // tile t: problem t / (n_rb n_cols), then column tile, then row block (the
  // CTAs running at once share a U tile in L2)
  const int per = n_rb * n_cols;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* ring = base;                              // kStages x (Dh, Dl, Uh, Ul)
  uint8_t* Wbuf = base + kStages * kStage;           // kWBufs half tiles
  Smem* sm = reinterpret_cast<Smem*>(Wbuf + kWBufs * kWHalf);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&sm->full[i], 1);
      mbar_init(&sm->empty[i], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&sm->acc_full[a], 1);
      mbar_init(&sm->acc_empty[a], 128);
    }
    for (int w = 0; w < kWBufs; ++w) {
      mbar_init(&sm->w_full[w], 1);
      mbar_init(&sm->w_written[w], 128);
      mbar_init(&sm->w_empty[w], 1);
    }
    mbar_init(&sm->drain, 1);
    sm->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&sm->tmem_base, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm->tmem_base;
  pdl_wait();

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer
    tma_prefetch(&tmDh);
    tma_prefetch(&tmDl);
    tma_prefetch(&tmUh);
    tma_prefetch(&tmUl);
    tma_prefetch(&tmW);
    const uint64_t keep_pol = policy_evict_last();
    const uint64_t w_pol = keep_w ? keep_pol : policy_evict_first();
    int s = 0, issued = 0, hw = 0;   // hw: W~ halves issued
    uint32_t ph = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < n_tiles && !aborted(sm); t += gridDim.x) {
      const int pb = t / per, rb = (t % per) % n_rb, tn = (t % per) / n_rb;
      for (int h = 0; h < 2; ++h, ++hw) {   // the W~ tile first: the long HBM latency
        const int wb = hw % kWBufs;
        if (!mbar_wait(&sm->w_empty[wb], ((hw / kWBufs) & 1) ^ 1)) {
          give_up(sm, status);
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&sm->w_full[wb], kWHalf);
        for (int q = 0; q < 2; ++q)
          tma_load_3d_hint(Wbuf + wb * kWHalf + q * kWBox, &tmW, &sm->w_full[wb],
                           e + tn * UN + h * 32 + q * WBOX, rb * UM, pb, w_pol);
      }
      for (int kk = 0; ok && kk < nkb * kNChunks; ++kk) {
        const int kx = kofs + kk * KC;   // K coordinate of this chunk
        if (!mbar_wait(&sm->empty[s], ph ^ 1)) {
          give_up(sm, status);
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&sm->full[s], kStage);
        uint8_t* st = ring + s * kStage;
        tma_load_3d_hint(st, &tmDh, &sm->full[s], kx, rb * UM, pb, keep_pol);
        tma_load_3d_hint(st + kAPart, &tmDl, &sm->full[s], kx, rb * UM, pb, keep_pol);
        tma_load_3d_hint(st + 2 * kAPart, &tmUh, &sm->full[s], kx, e + tn * UN, pb, keep_pol);
        tma_load_3d_hint(st + 2 * kAPart + kBPart, &tmUl, &sm->full[s], kx, e + tn * UN, pb,
                         keep_pol);
        ++issued;
        if (++s == kStages) {
          s = 0;
          ph ^= 1;
        }
      }
    }
    if (aborted(sm)) {   // let issued copies land before the CTA exits
      for (int k = 0; k < kStages && k < issued; ++k) {
        if (--s < 0) {
          s = kStages - 1;
          ph ^= 1;
        }
        mbar_wait_drain(&sm->full[s], ph);
      }
      for (int k = 1; k <= kWBufs && k <= hw; ++k)
        mbar_wait_drain(&sm->w_full[(hw - k) % kWBufs], ((hw - k) / kWBufs) & 1);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc = instr_desc(2 /*tf32*/, 0, 0 /*both K-major*/, UM, UN);
    int s = 0, lt = 0;
    uint32_t ph = 0;
    bool ok = true;
    // one accumulator round per 128-deep K block of a tile; lt counts rounds
    for (int t = blockIdx.x; ok && t < n_tiles && !aborted(sm); t += gridDim.x)
     for (int kb = 0; ok && kb < nkb; ++kb, ++lt) {
      const int buf = lt & 1;
      if (!mbar_wait(&sm->acc_empty[buf], ((lt >> 1) & 1) ^ 1)) {
        give_up(sm, status);
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t acc = tmem + buf * kBufCols;
      for (int kc = 0; kc < kNChunks; ++kc) {
        if (!mbar_wait(&sm->full[s], ph)) {
          give_up(sm, status);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t ah = smem_u32(ring + s * kStage), al = ah + kAPart;
        const uint32_t bh = ah + 2 * kAPart, bl = bh + kBPart;
        const uint32_t mainc = acc + (kc >> 1) * UN, cross = acc + 2 * UN;
#pragma unroll
        for (int k = 0; k < KC / 8; ++k) {
          const uint64_t dah = smem_desc_sw128(ah + 32 * k, 16, 1024);
          const uint64_t dal = smem_desc_sw128(al + 32 * k, 16, 1024);
          const uint64_t dbh = smem_desc_sw128(bh + 32 * k, 16, 1024);
          const uint64_t dbl = smem_desc_sw128(bl + 32 * k, 16, 1024);
          mma_tf32(mainc, dah, dbh, idesc, (kc & 1) | k);
          mma_tf32(cross, dah, dbl, idesc, kc | k);
          mma_tf32(cross, dal, dbh, idesc, 1);
        }
        mma_commit(&sm->empty[s]);
        if (++s == kStages) {
          s = 0;
          ph ^= 1;
        }
      }
      if (!ok) break;
      mma_commit(&sm->acc_full[buf]);
    }
    mma_commit(&sm->drain);
    mbar_wait_drain(&sm->drain, 0);
  } else if (warp >= 2 && warp < 6) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int r = q * 32 + lane;        // tile row = TMEM lane
    int lt = 0, ht = 0;   // lt: accumulator rounds, ht: tiles (W~ halves 2 ht, 2 ht + 1)
    bool ok = true;
    for (int t = blockIdx.x; ok && t < n_tiles && !__any_sync(0xffffffffu, aborted(sm));
         t += gridDim.x, ++ht)
     for (int kb = 0; ok && kb < nkb; ++kb, ++lt) {
      const int buf = lt & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&sm->acc_full[buf], (lt >> 1) & 1))) {
        give_up(sm, status);
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t ta = tmem + ((uint32_t)(q * 32) << 16) + buf * kBufCols;
      for (int h = 0; h < 2; ++h) {
        const int hw = 2 * ht + h, wb = hw % kWBufs;
        const uint32_t wpar = (hw / kWBufs) & 1;
        float m0[32], m1[32], cr[32];
        tmem_ld32(ta + h * 32, m0);
        tmem_ld32(ta + UN + h * 32, m1);
        tmem_ld32(ta + 2 * UN + h * 32, cr);
        if (kb == 0 && !__all_sync(0xffffffffu, mbar_wait(&sm->w_full[wb], wpar))) {
          give_up(sm, status);
          ok = false;
          break;
        }
#pragma unroll
        for (int qb = 0; qb < 2; ++qb) {
          uint8_t* rowp = Wbuf + wb * kWHalf + qb * kWBox + r * 128;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            double2* w = reinterpret_cast<double2*>(rowp + ((j ^ (r & 7)) << 4));
            const int c = qb * WBOX + 2 * j;
            double2 x = *w;
            x.x -= ((double)m0[c] + (double)m1[c]) + (double)cr[c];
            x.y -= ((double)m0[c + 1] + (double)m1[c + 1]) + (double)cr[c + 1];
            *w = x;
          }
        }
        if (kb == nkb - 1) {   // the tile's last K block: hand the half to the store
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          mbar_arrive(&sm->w_written[wb]);
        }
      }
      tc_fence_before();
      mbar_arrive(&sm->acc_empty[buf]);
    }
  } else if (warp == 6 && lane == 0) {
    // ------------------------------------------------------------ store
    const uint64_t w_pol = keep_w ? policy_evict_last() : policy_evict_first();
    int hw = 0, prev = -1;
    for (int t = blockIdx.x; t < n_tiles && !aborted(sm); t += gridDim.x) {
      const int pb = t / per, rb = (t % per) % n_rb, tn = (t % per) / n_rb;
      bool ok = true;
      for (int h = 0; h < 2; ++h, ++hw) {
        const int wb = hw % kWBufs;
        if (!mbar_wait(&sm->w_written[wb], (hw / kWBufs) & 1)) {
          give_up(sm, status);
          ok = false;
          break;
        }
        for (int qb = 0; qb < 2; ++qb)
          tma_store_3d(&tmW, Wbuf + wb * kWHalf + qb * kWBox, e + tn * UN + h * 32 + qb * WBOX,
                       rb * UM, pb, w_pol);
        bulk_commit();
        bulk_wait_read_all_but_one();   // the previous half's store has read its buffer
        if (prev >= 0) mbar_arrive(&sm->w_empty[prev]);
        prev = wb;
      }
      if (!ok) break;
    }
    bulk_wait_all();
    if (prev >= 0) mbar_arrive(&sm->w_empty[prev]);
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

// 3-D map (columns, rows, problem): rows ld elements apart, problems
// `stride` elements apart.
static bool map3(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize,
                 int64_t cols, int64_t rows, int64_t ld, int P, int64_t stride, uint32_t box0,
                 uint32_t box1) {
  const uint64_t dims[3] = {(uint64_t)cols, (uint64_t)rows, (uint64_t)P};
  const uint64_t strides[2] = {(uint64_t)ld * esize, (uint64_t)stride * esize};
  const uint32_t box[3] = {box0, box1, 1u};
  return encode_tmap_nd(m, base, dt, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

bool make_update_maps(UpdateMaps* m, const float* Dh, const float* Dl, const float* Uh,
                      const float* Ul, const double* Wt, int64_t d_out, int64_t d_in,
                      int64_t kcols, int P) {
  constexpr CUtensorMapDataType F32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  return map3(&m->Dh, Dh, F32, 4, kcols, d_out, kcols, P, d_out * kcols, KC, UM) &&
         map3(&m->Dl, Dl, F32, 4, kcols, d_out, kcols, P, d_out * kcols, KC, UM) &&
         map3(&m->Uh, Uh, F32, 4, kcols, d_in, kcols, P, d_in * kcols, KC, UN) &&
         map3(&m->Ul, Ul, F32, 4, kcols, d_in, kcols, P, d_in * kcols, KC, UN) &&
         map3(&m->W, Wt, CU_TENSOR_MAP_DATA_TYPE_FLOAT64, 8, d_in, d_out, d_in, P, d_out * d_in,
              WBOX, UM);
}

nvfp4_status launch_update_tc(const UpdateMaps& m, int64_t d_out, int64_t d_in, int64_t e,
                              int64_t e_end, int kofs, int nkb, bool keep_w, int P, int* status,
                              cudaStream_t st) {
  const int n = (int)(e_end - e);
  if (n <= 0 || d_out <= 0 || nkb <= 0 || P < 1) return NVFP4_OK;
  // a tile may not reach past e_end unless e_end is the last column (the
  // tensor map clips there): tiles are UN columns wide
  if (e_end < d_in && n % UN != 0) return NVFP4_ERR_INVALID_ARG;
  const int n_rb = (int)((d_out + UM - 1) / UM);
  const int n_cols = (n + UN - 1) / UN;
  const int n_tiles = n_rb * n_cols * P;
  const int sms = num_sms();
  NVFP4_CUDA_TRY(cudaFuncSetAttribute(update_tc_kernel,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem));
  NVFP4_CUDA_TRY(launch_chained(update_tc_kernel, dim3(n_tiles < sms ? n_tiles : sms),
                                dim3(kThreads), kSmem, st, m.Dh, m.Dl, m.Uh, m.Ul, m.W, (int)e,
                                n_rb, n_cols, n_tiles, kofs, nkb, keep_w ? 1 : 0, status));
  count_launches(1);
  return NVFP4_OK;
}

}  // namespace nvfp4

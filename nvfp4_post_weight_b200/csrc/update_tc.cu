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
// and subtracts the sum from W~ in place.
//
// Both operands are K-major (Uh/Ul hold the batch's rows of U transposed,
// 128 K values per column), in the canonical 128-byte-swizzled layout.
//
// Persistent CTA per SM, warp-specialised:
//   warp 0     TMA producer: the CTA's 128-row slice of Dh/Dl (all of K,
//              128 KB, resident while the CTA walks its column tiles), a
//              2-stage ring of (Uh, Ul) chunks of 64 columns x 32 K values, and
//              the W~ tile itself (128 rows x 64 fp64, as two 32-column halves
//              in two 32 KB buffers, 128-byte swizzled)
//   warp 1     MMA issuer, 12 MMAs (M=128, N=64, K=8) per K chunk
//   warps 2-5  epilogue: per half tile, TMEM -> registers, W~ -= sum in the
//              shared-memory buffer, then one thread writes the half back with
//              a TMA store and frees the buffer once the store has read it.
//   The W~ traffic (the roofline of this kernel) is all bulk asynchronous.
// Work item = (128-row block, one of P interleaved column-tile sets).
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
constexpr uint32_t kAChunk = UM * KC * 4;      // 16 KB (hi or lo)
constexpr uint32_t kABytes = 2 * kNChunks * kAChunk;   // 128 KB
constexpr uint32_t kBHalf = UN * KC * 4;       // 64 columns x 128 B = 8 KB (hi or lo)
constexpr uint32_t kBStage = 2 * kBHalf;       // 16 KB
constexpr int kBStages = 2;
constexpr int WBOX = 16;                       // fp64 per TMA box row (128 B)
constexpr uint32_t kWBox = UM * WBOX * 8;      // 16 KB
constexpr uint32_t kWHalf = 2 * kWBox;         // 32 columns = 32 KB
constexpr int kThreads = 192;
constexpr uint32_t kAccCols = 3 * UN;          // main0, main1, cross
constexpr uint32_t kBufCols = 256;             // TMEM columns between the two buffers
constexpr uint32_t kTmemCols = 512;
constexpr size_t kSmem = kABytes + kBStages * kBStage + 2 * kWHalf + 1024 + 256;

struct Smem {
  uint64_t a_full, a_empty;
  uint64_t b_full[kBStages], b_empty[kBStages];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t w_full[2], w_written[2], w_empty[2];
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

// TMA tile store from shared memory (out-of-range parts are not written).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int c0,
                                             int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(map),
      "r"(smem_u32(src)), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read() {   // sources of all committed stores read
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() {    // all committed stores complete
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

__global__ void __launch_bounds__(kThreads, 1)
    update_tc_kernel(const __grid_constant__ CUtensorMap tmDh,
                     const __grid_constant__ CUtensorMap tmDl,
                     const __grid_constant__ CUtensorMap tmUh,
                     const __grid_constant__ CUtensorMap tmUl,
                     const __grid_constant__ CUtensorMap tmW, double* __restrict__ Wt,
                     int64_t ldw, int d_out, int n, int e, int n_rb, int n_nt, int parts,
                     int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* A = base;                      // hi chunks 0..3, then lo chunks 0..3
  uint8_t* Bring = base + kABytes;
  uint8_t* Wbuf = Bring + kBStages * kBStage;   // two half-tile buffers
  Smem* sm = reinterpret_cast<Smem*>(Wbuf + 2 * kWHalf);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int items = n_rb * parts;

  if (threadIdx.x == 0) {
    mbar_init(&sm->a_full, 1);
    mbar_init(&sm->a_empty, 1);
    for (int s = 0; s < kBStages; ++s) {
      mbar_init(&sm->b_full[s], 1);
      mbar_init(&sm->b_empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&sm->acc_full[a], 1);
      mbar_init(&sm->acc_empty[a], 128);
      mbar_init(&sm->w_full[a], 1);
      mbar_init(&sm->w_written[a], 128);
      mbar_init(&sm->w_empty[a], 1);
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

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer
    tma_prefetch(&tmDh);
    tma_prefetch(&tmDl);
    tma_prefetch(&tmUh);
    tma_prefetch(&tmUl);
    tma_prefetch(&tmW);
    int s = 0, it = 0, issued = 0, wt = 0;
    uint32_t ph = 0;
    bool ok = true;
    int a_armed = -1;   // last A load armed, to drain on abort
    for (int item = blockIdx.x; ok && item < items && !aborted(sm); item += gridDim.x, ++it) {
      const int rb = item % n_rb, p = item / n_rb;
      if (!mbar_wait(&sm->a_empty, (it & 1) ^ 1)) {
        give_up(sm, status);
        break;
      }
      mbar_arrive_expect_tx(&sm->a_full, kABytes);
      for (int kc = 0; kc < kNChunks; ++kc) {
        tma_load_2d(A + kc * kAChunk, &tmDh, &sm->a_full, kc * KC, rb * UM);
        tma_load_2d(A + (kNChunks + kc) * kAChunk, &tmDl, &sm->a_full, kc * KC, rb * UM);
      }
      a_armed = it;
      for (int tn = p; ok && tn < n_nt; tn += parts) {
        for (int kc = 0; kc < kNChunks; ++kc) {
          if (!mbar_wait(&sm->b_empty[s], ph ^ 1)) {
            give_up(sm, status);
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&sm->b_full[s], kBStage);
          uint8_t* st = Bring + s * kBStage;
          tma_load_2d(st, &tmUh, &sm->b_full[s], kc * KC, e + tn * UN);
          tma_load_2d(st + kBHalf, &tmUl, &sm->b_full[s], kc * KC, e + tn * UN);
          ++issued;
          if (++s == kBStages) {
            s = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
        for (int h = 0; h < 2; ++h) {   // the W~ tile, as two 32-column halves
          if (!mbar_wait(&sm->w_empty[h], (wt & 1) ^ 1)) {
            give_up(sm, status);
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&sm->w_full[h], kWHalf);
          for (int q = 0; q < 2; ++q)
            tma_load_2d(Wbuf + h * kWHalf + q * kWBox, &tmW, &sm->w_full[h],
                        e + tn * UN + h * 32 + q * WBOX, rb * UM);
        }
        ++wt;
      }
    }
    if (aborted(sm)) {   // let issued copies land before the CTA exits
      if (a_armed >= 0) mbar_wait(&sm->a_full, a_armed & 1);
      for (int k = 0; k < kBStages && k < issued; ++k) {
        if (--s < 0) {
          s = kBStages - 1;
          ph ^= 1;
        }
        mbar_wait(&sm->b_full[s], ph);
      }
      if (wt > 0)
        for (int h = 0; h < 2; ++h) mbar_wait(&sm->w_full[h], (wt - 1) & 1);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc = instr_desc(2 /*tf32*/, 0, 0 /*both K-major*/, UM, UN);
    int s = 0, it = 0, lt = 0;
    uint32_t ph = 0;
    bool ok = true;
    const uint32_t a0 = smem_u32(A);
    for (int item = blockIdx.x; ok && item < items && !aborted(sm); item += gridDim.x, ++it) {
      const int p = item / n_rb;
      if (!mbar_wait(&sm->a_full, it & 1)) {
        give_up(sm, status);
        break;
      }
      tc_fence_after();
      for (int tn = p; ok && tn < n_nt; tn += parts, ++lt) {
        const int buf = lt & 1;
        if (!mbar_wait(&sm->acc_empty[buf], ((lt >> 1) & 1) ^ 1)) {
          give_up(sm, status);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t acc = tmem + buf * kBufCols;
        for (int kc = 0; kc < kNChunks; ++kc) {
          if (!mbar_wait(&sm->b_full[s], ph)) {
            give_up(sm, status);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t ah = a0 + kc * kAChunk, al = a0 + (kNChunks + kc) * kAChunk;
          const uint32_t bh = smem_u32(Bring + s * kBStage), bl = bh + kBHalf;
          const uint32_t main = acc + (kc >> 1) * UN, cross = acc + 2 * UN;
#pragma unroll
          for (int k = 0; k < KC / 8; ++k) {
            const uint64_t dah = smem_desc_sw128(ah + 32 * k, 16, 1024);
            const uint64_t dal = smem_desc_sw128(al + 32 * k, 16, 1024);
            const uint64_t dbh = smem_desc_sw128(bh + 32 * k, 16, 1024);
            const uint64_t dbl = smem_desc_sw128(bl + 32 * k, 16, 1024);
            mma_tf32(main, dah, dbh, idesc, (kc & 1) | k);
            mma_tf32(cross, dah, dbl, idesc, kc | k);
            mma_tf32(cross, dal, dbh, idesc, 1);
          }
          mma_commit(&sm->b_empty[s]);
          if (++s == kBStages) {
            s = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
        mma_commit(&sm->acc_full[buf]);
      }
      if (ok) mma_commit(&sm->a_empty);
    }
    mma_commit(&sm->drain);
    mbar_wait(&sm->drain, 0);
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int r = q * 32 + lane;        // tile row = TMEM lane
    const bool storer = threadIdx.x == 64;
    int lt = 0;
    bool ok = true;
    for (int item = blockIdx.x; ok && item < items && !__any_sync(0xffffffffu, aborted(sm));
         item += gridDim.x) {
      const int rb = item % n_rb, p = item / n_rb;
      for (int tn = p; ok && tn < n_nt; tn += parts, ++lt) {
        const int buf = lt & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&sm->acc_full[buf], (lt >> 1) & 1))) {
          give_up(sm, status);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t ta = tmem + ((uint32_t)(q * 32) << 16) + buf * kBufCols;
        for (int h = 0; h < 2; ++h) {
          float m0[32], m1[32], cr[32];
          tmem_ld32(ta + h * 32, m0);
          tmem_ld32(ta + UN + h * 32, m1);
          tmem_ld32(ta + 2 * UN + h * 32, cr);
          if (!__all_sync(0xffffffffu, mbar_wait(&sm->w_full[h], lt & 1))) {
            give_up(sm, status);
            ok = false;
            break;
          }
          // row r of the half: two 128-byte box rows, 16-byte chunk j stored at
          // position j ^ (r % 8) (the 128-byte swizzle)
#pragma unroll
          for (int qb = 0; qb < 2; ++qb) {
            uint8_t* rowp = Wbuf + h * kWHalf + qb * kWBox + r * 128;
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
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          mbar_arrive(&sm->w_written[h]);
          if (storer) {
            // all 128 rows written -> store the half back, free the buffer once
            // the store has read it
            if (!mbar_wait(&sm->w_written[h], lt & 1)) {
              give_up(sm, status);
            } else {
              for (int qb = 0; qb < 2; ++qb)
                tma_store_2d(&tmW, Wbuf + h * kWHalf + qb * kWBox,
                             e + tn * UN + h * 32 + qb * WBOX, rb * UM);
              bulk_commit();
              bulk_wait_read();
            }
            mbar_arrive(&sm->w_empty[h]);
          }
        }
        tc_fence_before();
        mbar_arrive(&sm->acc_empty[buf]);
      }
    }
    if (storer) bulk_wait_all();   // the last stores complete before the CTA exits
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

bool make_update_maps(UpdateMaps* m, const float* Dh, const float* Dl, const float* Uh,
                      const float* Ul, const double* Wt, int64_t d_out, int64_t d_in) {
  const uint64_t dw[2] = {(uint64_t)d_in, (uint64_t)d_out};
  const uint64_t sw[1] = {(uint64_t)d_in * 8};
  const uint32_t bw[2] = {(uint32_t)WBOX, (uint32_t)UM};
  const uint64_t da[2] = {(uint64_t)UK, (uint64_t)d_out};
  const uint64_t sa[1] = {(uint64_t)UK * 4};
  const uint32_t ba[2] = {(uint32_t)KC, (uint32_t)UM};
  const uint64_t db[2] = {(uint64_t)UK, (uint64_t)d_in};
  const uint64_t sb[1] = {(uint64_t)UK * 4};
  const uint32_t bb[2] = {(uint32_t)KC, (uint32_t)UN};
  return encode_tmap_2d(&m->Dh, Dh, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, da, sa, ba,
                        CU_TENSOR_MAP_SWIZZLE_128B) &&
         encode_tmap_2d(&m->Dl, Dl, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, da, sa, ba,
                        CU_TENSOR_MAP_SWIZZLE_128B) &&
         encode_tmap_2d(&m->Uh, Uh, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, db, sb, bb,
                        CU_TENSOR_MAP_SWIZZLE_128B) &&
         encode_tmap_2d(&m->Ul, Ul, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, db, sb, bb,
                        CU_TENSOR_MAP_SWIZZLE_128B) &&
         encode_tmap_2d(&m->W, Wt, CU_TENSOR_MAP_DATA_TYPE_FLOAT64, dw, sw, bw,
                        CU_TENSOR_MAP_SWIZZLE_128B);
}

nvfp4_status launch_update_tc(const UpdateMaps& m, double* Wt, int64_t ldw, int64_t d_out,
                              int64_t d_in, int64_t e, int* status, cudaStream_t st) {
  const int n = (int)(d_in - e);
  if (n <= 0 || d_out <= 0) return NVFP4_OK;
  const int n_rb = (int)((d_out + UM - 1) / UM);
  const int n_nt = (n + UN - 1) / UN;
  const int sms = num_sms();
  int parts = n_rb >= sms ? 1 : sms / n_rb;
  if (parts > n_nt) parts = n_nt;
  if (parts < 1) parts = 1;
  const int items = n_rb * parts;
  NVFP4_CUDA_TRY(cudaFuncSetAttribute(update_tc_kernel,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem));
  update_tc_kernel<<<items < sms ? items : sms, kThreads, kSmem, st>>>(
      m.Dh, m.Dl, m.Uh, m.Ul, m.W, Wt, ldw, (int)d_out, n, (int)e, n_rb, n_nt, parts, status);
  NVFP4_LAUNCH_CHECK();
  count_launches(1);
  return NVFP4_OK;
}

}  // namespace nvfp4

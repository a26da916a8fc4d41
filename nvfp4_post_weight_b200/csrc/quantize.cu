// a5-a8: global scale, working copy, Schur Replay block-scale selection inside
// GPTQ, and the lazy-batch trailing update.
//
// "Replay the Curvature" (arXiv 2609.36654v1), Abstract: GPTQ quantizes the
// columns in order and each quantized column updates the columns after it, so
// a block scale changes the values the rest of its block is quantized from.
// Schur Replay scores every candidate scale by replaying those in-block
// updates and measuring the block error that remains after compensation from
// the still-unquantized columns; the best candidate is kept.
//
// With U the upper factor of H_d^-1 (H_d^-1 = U^T U), quantizing column j of
// a row leaves delta_j = (v_j - q_j) / U_jj and the later columns absorb
// delta_j * U[j, i].  delta_j^2 = (v_j - q_j)^2 / U_jj^2 where 1/U_jj^2 is the
// Schur complement of column j given the columns after it, and the block's
// sum of delta_j^2 is its exact share of tr((W-Q) H_d (W-Q)^T).
//
// Precision: the working copy W~ is kept in fp64 and the replay runs in fp64.
// The codes are discrete decisions (nearest E2M1 value, argmin over scales)
// and one flipped code changes every later update of its row, so the values
// they are taken on must carry more than fp32's 24 bits; the factor U itself
// is fp32 (its rounding moves no decision on the workloads measured).
//
// Layout of the work: columns go in lazy batches of 128.  For one batch the
// replay kernel walks the batch's 8 blocks for every row (a half-warp per row,
// lane = candidate scale) with the row's 128 batch values in shared memory,
// and applies each chosen block's deltas to the rest of the batch; it writes
// the batch's deltas as tf32 hi/lo pairs.  The trailing update W~[:, e:] -=
// Delta U[batch, e:] is two-level (super_width below): each batch updates
// the rest of its super-batch at once (update_tc), and each super-batch
// updates every column beyond it with K = 1024 (the 3xTF32 GEMM on the same
// hi/lo pairs of Delta and of U's rows).
#include <math.h>

#include "common.cuh"
#include "nvfp4_format.cuh"
#include "sm100.cuh"

namespace nvfp4 {
namespace {

struct QuantHeader {   // one per problem of a group
  int status;
  unsigned amax_bits;  // max |W| as fp32 bits (non-negative floats order as uints)
};

// The caller's buffers of every problem of a group, written into the group
// region once per call (init_group_kernel) and read by the kernels.
struct QuantTable {
  const void* W[kMaxGroup];
  const float* U[kMaxGroup];
  const uint8_t* dead[kMaxGroup];
  uint8_t* codes[kMaxGroup];
  uint8_t* scales[kMaxGroup];
  float* sg[kMaxGroup];
  double* err[kMaxGroup];
  const float* amax_in[kMaxGroup];
};

// Columns per super-batch.  Inside a super-batch every lazy batch updates only
// the super-batch's later columns (an fp64 W~ slab of d_out x 1024 that stays
// in L2); the super-batch's deltas reach the columns beyond it in one update
// with K = 1024, so the HBM-resident rest of W~ is read and written once per
// super-batch instead of once per batch.  Narrow layers keep one batch per
// super-batch (the plain lazy-batch scheme).
int64_t super_width(int64_t d_in) { return d_in >= 2048 ? 8 * kLazyBatch : kLazyBatch; }

// A group region of the quantize: the group header (its first int the status
// word), the pointer table, P problem headers, then P copies each (uniform
// strides) of the arrays below.
struct QuantLayout {
  int* gstatus;
  QuantTable* tab;
  QuantHeader* hdr;
  int64_t S;       // super-batch width (K values per row of the four below)
  double* Wt;      // d_out x d_in working copy (stride d_out d_in)
  float* Dh;       // d_out x S: the super-batch's deltas, tf32-rounded part
  float* Dl;       // d_out x S: remainder (delta - Dh)
  float* Uh;       // d_in x S: the super-batch's rows of U transposed, tf32 part
  float* Ul;       // d_in x S: remainder
  double* rowerr;  // d_out
};

size_t quant_group_bytes(int64_t d_out, int64_t d_in, int P) {
  const int64_t S = super_width(d_in);
  return kWsHeader + align256(sizeof(QuantTable)) + align256(sizeof(QuantHeader) * P) +
         align256(sizeof(double) * d_out * d_in * P) + 2 * align256(sizeof(float) * d_out * S * P) +
         2 * align256(sizeof(float) * S * d_in * P) + align256(sizeof(double) * d_out * P);
}

QuantLayout quant_layout(void* ws, int64_t d_out, int64_t d_in, int P) {
  char* p = static_cast<char*>(ws);
  QuantLayout L;
  L.gstatus = reinterpret_cast<int*>(p);
  L.S = super_width(d_in);
  size_t off = kWsHeader;
  L.tab = reinterpret_cast<QuantTable*>(p + off);
  off += align256(sizeof(QuantTable));
  L.hdr = reinterpret_cast<QuantHeader*>(p + off);
  off += align256(sizeof(QuantHeader) * P);
  L.Wt = reinterpret_cast<double*>(p + off);
  off += align256(sizeof(double) * d_out * d_in * P);
  L.Dh = reinterpret_cast<float*>(p + off);
  off += align256(sizeof(float) * d_out * L.S * P);
  L.Dl = reinterpret_cast<float*>(p + off);
  off += align256(sizeof(float) * d_out * L.S * P);
  L.Uh = reinterpret_cast<float*>(p + off);
  off += align256(sizeof(float) * L.S * d_in * P);
  L.Ul = reinterpret_cast<float*>(p + off);
  off += align256(sizeof(float) * L.S * d_in * P);
  L.rowerr = reinterpret_cast<double*>(p + off);
  return L;
}

// Clears the group's status word and problem headers and stores the pointer
// table (one CTA).
__global__ void init_group_kernel(QuantTable t, QuantTable* dst, int* gstatus, QuantHeader* hdr,
                                  int P) {
  if (threadIdx.x == 0) *gstatus = 0;
  for (int i = threadIdx.x; i < P; i += blockDim.x) hdr[i] = QuantHeader{0, 0u};
  const uint64_t* src = reinterpret_cast<const uint64_t*>(&t);
  uint64_t* out = reinterpret_cast<uint64_t*>(dst);
  for (int i = threadIdx.x; i < (int)(sizeof(QuantTable) / 8); i += blockDim.x) out[i] = src[i];
}

// a5 + a6: W~ = fp64(W) with dead columns zeroed, amax |W~|, non-finite check.
// Eight consecutive elements per thread step (d_in is a multiple of 16);
// problem blockIdx.y of the group.
template <typename T>
__global__ void wprep_kernel(const QuantTable* __restrict__ tab, int64_t d_out, int64_t d_in,
                             double* __restrict__ Wt, double* __restrict__ rowerr,
                             QuantHeader* hdrs, int* gstatus) {
  const int pb = blockIdx.y;
  const T* __restrict__ W = static_cast<const T*>(tab->W[pb]);
  const uint8_t* __restrict__ dead = tab->dead[pb];
  QuantHeader* hdr = hdrs + pb;
  Wt += pb * d_out * d_in;
  rowerr += pb * d_out;
  const int64_t n8 = d_out * d_in / 8;
  float m = 0.f;
  bool bad = false;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8;
       i += (int64_t)gridDim.x * blockDim.x) {
    float v[8];
    if constexpr (sizeof(T) == 2) {
      const uint4 raw = reinterpret_cast<const uint4*>(W)[i];
      const uint32_t u[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        v[2 * k] = __uint_as_float(u[k] << 16);
        v[2 * k + 1] = __uint_as_float(u[k] & 0xffff0000u);
      }
    } else {
      const float4 a = reinterpret_cast<const float4*>(W)[2 * i];
      const float4 b = reinterpret_cast<const float4*>(W)[2 * i + 1];
      v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
      v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
    if (dead) {
      const int64_t c = (i * 8) % d_in;
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (dead[c + k]) v[k] = 0.f;
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      bad |= !isfinite(v[k]);
      m = fmaxf(m, fabsf(v[k]));
    }
    double2* o = reinterpret_cast<double2*>(Wt + 8 * i);
#pragma unroll
    for (int k = 0; k < 4; ++k) o[k] = make_double2(v[2 * k], v[2 * k + 1]);
  }
  for (int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; r < d_out;
       r += (int64_t)gridDim.x * blockDim.x)
    rowerr[r] = 0.0;
  if (__any_sync(0xffffffffu, bad)) {
    if ((threadIdx.x & 31) == 0) {
      flag_status(&hdr->status, NVFP4_ERR_NONFINITE);
      flag_status(gstatus, NVFP4_ERR_NONFINITE);
    }
  }
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) atomicMax(&hdr->amax_bits, __float_as_uint(m));
}

// s_g = amax / (6 * 448) correctly rounded to fp32, 1 when W == 0; amax is
// this call's own max |W~| unless the caller gives the layer's (row shards).
// One thread per problem of the group.
__global__ void global_scale_kernel(const QuantTable* __restrict__ tab, const QuantHeader* hdrs,
                                    int P) {
  const int pb = threadIdx.x;
  if (pb >= P) return;
  const float* amax_in = tab->amax_in[pb];
  const float amax = amax_in ? *amax_in : __uint_as_float(hdrs[pb].amax_bits);
  *tab->sg[pb] = amax > 0.f ? __fdiv_rn(amax, 2688.0f) : 1.0f;
}

// max |W| (dead columns as 0) into *amax_bits (fp32 bits; non-negative floats
// order as unsigned integers), which the caller zeroed.
template <typename T>
__global__ void weight_amax_kernel(const T* __restrict__ W, int64_t d_out, int64_t d_in,
                                   const uint8_t* __restrict__ dead,
                                   unsigned* __restrict__ amax_bits) {
  const int64_t n = d_out * d_in;
  float m = 0.f;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    float v;
    if constexpr (sizeof(T) == 2)
      v = __uint_as_float((uint32_t)W[i] << 16);
    else
      v = W[i];
    if (dead && dead[i % d_in]) v = 0.f;
    m = fmaxf(m, fabsf(v));
  }
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) atomicMax(amax_bits, __float_as_uint(m));
}

// 14 warps = 28 rows in flight, one CTA per SM: 4096 rows fill 147 SMs
// evenly (16-row CTAs two to an SM would leave some SMs 32 rows, others 16)
constexpr int kReplayThreads = 448;
constexpr int kRowsPerCta = kReplayThreads / 16;
constexpr int kNb = kLazyBatch / kBlock;            // blocks per batch (8)
constexpr int kUTiles = kNb * (kNb + 1) / 2;        // upper 16x16 tiles of a batch (36)

// Index of the upper tile (p, q), q >= p, in the packed tile array.
__device__ __forceinline__ int utile(int p, int q) { return p * (2 * kNb - 1 - p) / 2 + q; }

// The super-batch's rows k < nk of U, transposed (S values per row, K
// contiguous: the updates' B operand), for the columns j >= j0, split as
// Uh[j][k] + Ul[j][k] = U[cs + k][j] (tf32 part and remainder): the per-batch
// updates read the super-batch's own columns, the super-batch update the
// columns beyond it.  32 x 32 tiles transposed through shared memory.
// Problem blockIdx.z of the group.
__global__ void __launch_bounds__(256) split_u_rows_kernel(const QuantTable* __restrict__ tab,
                                                           int64_t d_in, int64_t cs, int nk,
                                                           int64_t j0, int64_t S,
                                                           float* __restrict__ Uh,
                                                           float* __restrict__ Ul) {
  __shared__ float t[32][33];
  pdl_wait();
  const float* __restrict__ U = tab->U[blockIdx.z];
  Uh += blockIdx.z * d_in * S;
  Ul += blockIdx.z * d_in * S;
  const int64_t jb = j0 + (int64_t)blockIdx.x * 32;
  const int k0 = blockIdx.y * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  for (int r = ty; r < 32; r += 8) {
    const int64_t j = jb + tx;
    t[r][tx] = (j < d_in && k0 + r < nk) ? U[(cs + k0 + r) * d_in + j] : 0.f;
  }
  __syncthreads();
  for (int r = ty; r < 32; r += 8) {
    const int64_t j = jb + r;
    if (j < d_in && k0 + tx < nk) {
      const float u = t[tx][r];
      const float h = sm100::tf32_rn(u);
      Uh[j * S + k0 + tx] = h;
      Ul[j * S + k0 + tx] = u - h;
    }
  }
}

// One candidate's replay of the in-block GPTQ updates (fp64).  v holds the
// block's 16 current values and is consumed.  Ud points at the block's
// diagonal 16x16 tile (row-major, 16-byte aligned), invd at its 1/U_jj.
// Returns the score sum delta_j^2; delta and the high words of the signed
// rounded magnitudes q_j / s are written out -- the code nibbles are derived
// once, from the winner's magnitudes, not by every candidate.
//
// The nearest E2M1 magnitude of |x| is taken by the add-and-subtract method
// (nvfp4_format.cuh) with the spacing constant picked, the saturation at 6
// and the sign applied on the high word of the double: every rounded value
// below 2^20 is a multiple of 1/2 whose low word is zero, so these integer
// steps give the same bits as the fp64 comparisons and selects they replace,
// and only the additions and the GPTQ arithmetic use the fp64 pipe.
__device__ __forceinline__ double replay(double (&v)[16], double s, double inv_s,
                                         const double* __restrict__ Ud,
                                         const double* __restrict__ invd, double (&dl)[16],
                                         uint32_t (&sq)[16]) {
  double score = 0.0;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const double x = __dmul_rn(v[j], inv_s);
    const uint32_t xh = (uint32_t)__double2hiint(x), xl = (uint32_t)__double2loint(x);
    const uint32_t ah = xh & 0x7FFFFFFFu;
    // 1.5 * 2^51, 2^52 or 2^53 for |x| below 2, below 4, from 4 up (spacing
    // 1/2, 1, 2)
    const int ex = (int)(ah >> 20) - 1023;
    const uint32_t mh = 0x43280000u + ((uint32_t)min(max(ex, 0), 2) << 20);
    const double M = __hiloint2double((int)mh, 0);
    const double r = __dsub_rn(__dadd_rn(__hiloint2double((int)ah, (int)xl), M), M);
    const bool neg = (xh >> 31) != 0 && (ah | xl) != 0;   // x < 0
    const uint32_t rh =
        min((uint32_t)__double2hiint(r), 0x40180000u /* 6.0 */) | (neg ? 0x80000000u : 0u);
    sq[j] = rh;
    const double sr = __hiloint2double((int)rh, 0);
    const double res = __fma_rn(-sr, s, v[j]);       // v_j - q_j, one rounding
    const double d = __dmul_rn(res, invd[j]);
    dl[j] = d;
    score = __fma_rn(d, d, score);
    // the later columns of the block absorb d: row j of the tile, two
    // values per 16-byte load
    const double2* Urow = reinterpret_cast<const double2*>(Ud + j * 16);
#pragma unroll
    for (int p = (j + 1) / 2; p < 8; ++p) {
      const double2 u = Urow[p];
      if (2 * p > j) v[2 * p] = __fma_rn(-d, u.x, v[2 * p]);
      v[2 * p + 1] = __fma_rn(-d, u.y, v[2 * p + 1]);
    }
  }
  return score;
}

// E2M1 code nibble of a rounded signed magnitude given by its high word (the
// form replay() writes): index 1 for 1/2, 2 (E - 1023) + 2 + m above it (E
// the biased exponent, m the mantissa's top bit), sign bit 8 for a negative
// nonzero value.
__device__ __forceinline__ uint32_t e2m1_nibble_hi(uint32_t rh) {
  const uint32_t mag = rh & 0x7FFFFFFFu, e = mag >> 20;
  const uint32_t idx = mag == 0 ? 0u : (e == 1022u ? 1u : 2u * (e - 1023u) + 2u + ((mag >> 19) & 1u));
  return idx | ((rh >> 31) && idx ? 8u : 0u);
}

// Block-scale rules: Schur Replay, and the two independent-block rules it is
// compared with ("Replay the Curvature", Abstract: a block evaluated on its own
// misestimates its final error): the amax scale k0, and the window code whose
// one-by-one rounding error of the block's values is smallest.  All three run
// the same GPTQ sweep; only the scale decision differs.
constexpr int kRuleSchurReplay = 0, kRuleAmax = 1, kRuleBlockMse = 2;

// One lazy batch of Schur Replay.  Half-warp = one row; lane hl = candidate hl
// of the current block.  The batch's upper block-triangular part of U lives in
// shared memory as 16x16 fp64 tiles, the rows' batch values next to it.
template <int kRule>
__global__ void __launch_bounds__(kReplayThreads)
    schur_replay_batch_kernel(const QuantTable* __restrict__ tab, double* __restrict__ Wt_all,
                              int64_t d_out, int64_t d_in, int c0, int bw,
                              float* __restrict__ Dh_all, float* __restrict__ Dl_all,
                              int64_t ldD, int kofs, double* __restrict__ rowerr_all) {
  extern __shared__ double4 smem_d4[];
  double* Ut = reinterpret_cast<double*>(smem_d4);           // kUTiles x 256
  double* invd = Ut + kUTiles * 256;                         // 128
  double* s_tab = invd + kLazyBatch;                         // e4m3_value(k) * s_g
  double* inv_tab = s_tab + 128;                             // 1 / s_tab[k]
  double* rows = inv_tab + 128;                              // kRowsPerCta x 128
  const int nblk = bw / kBlock;
  // problem blockIdx.y of the group: its buffers
  const int pb = blockIdx.y;
  const float* __restrict__ U = tab->U[pb];
  const float* __restrict__ sg_ptr = tab->sg[pb];
  double* __restrict__ Wt = Wt_all + (int64_t)pb * d_out * d_in;
  float* __restrict__ Dh = Dh_all + (int64_t)pb * d_out * ldD;
  float* __restrict__ Dl = Dl_all + (int64_t)pb * d_out * ldD;
  double* __restrict__ rowerr = rowerr_all + (int64_t)pb * d_out;
  uint8_t* __restrict__ codes = tab->codes[pb];
  uint8_t* __restrict__ scales = tab->scales[pb];
  pdl_wait();
  {
    // Stage the batch's upper block-triangular part of U as 16 x 16 fp64
    // tiles: thread t < 256 handles element e = t of every tile and issues
    // all its loads before any store.  The other threads fill the candidate
    // scale table (e4m3_value(k) s_g and its reciprocal) and 1/U_jj.
    static_assert(kReplayThreads >= 256 + 128, "tile elements, then the tables");
    if (threadIdx.x < 256) {
      const int e = threadIdx.x, i = e >> 4, j = e & 15;
      float u[kUTiles];
#pragma unroll
      for (int t = 0, p = 0, q = 0; t < kUTiles; ++t) {
        const int gi = 16 * p + i, gj = 16 * q + j;
        u[t] = (p < nblk && q < nblk && gj >= gi) ? U[(int64_t)(c0 + gi) * d_in + c0 + gj] : 0.f;
        if (++q == kNb) q = ++p;   // tiles (p, q), q >= p, row-major
      }
#pragma unroll
      for (int t = 0; t < kUTiles; ++t) Ut[t * 256 + e] = (double)u[t];
    } else {
      for (int c = threadIdx.x - 256; c < 128 + bw; c += kReplayThreads - 256) {
        if (c < 128) {
          const double sk = e4m3_value(c < 127 ? c : 126) * (double)*sg_ptr;
          s_tab[c] = sk;
          inv_tab[c] = 1.0 / sk;
        } else {
          const int jj = c - 128;
          invd[jj] = 1.0 / (double)U[(int64_t)(c0 + jj) * d_in + c0 + jj];
        }
      }
    }
  }
  __syncthreads();

  const double sg = (double)*sg_ptr;
  const double six_sg = 6.0 * sg;
  const int lane = threadIdx.x & 31, hl = lane & 15, half = lane >> 4;
  const int warp = threadIdx.x >> 5;
  const int rloc = warp * 2 + half;
  double* row = rows + rloc * kLazyBatch;
  uint32_t* mrow = reinterpret_cast<uint32_t*>(rows + kRowsPerCta * kLazyBatch) + rloc * 16;
  const unsigned FULL = 0xffffffffu;

  for (int64_t rb = (int64_t)blockIdx.x * kRowsPerCta; rb < d_out;
       rb += (int64_t)gridDim.x * kRowsPerCta) {
    const int64_t r = rb + rloc;
    const bool valid = r < d_out;
    // stage the row's batch values
    for (int c = hl; c < bw; c += 16) row[c] = valid ? Wt[r * d_in + c0 + c] : 0.0;
    __syncwarp();
    double rowsum = 0.0;

    for (int b = 0; b < nblk; ++b) {
      double v[16];
      double amax = 0.0;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        v[i] = row[16 * b + i];
        amax = fmax(amax, fabs(v[i]));
      }
      const int k0 = max(e4m3_code_rn(amax / six_sg), 1);
      const int lo = min(max(k0 - 8, 1), 127 - kCand);
      const double s = s_tab[lo + hl];   // e4m3_value * s_g, exact: 4 + 24 significant bits
      const double inv_s = inv_tab[lo + hl];
      const double* Ud = Ut + utile(b, b) * 256;
      const double* idb = invd + 16 * b;

      // the rule's selection score: the replay score itself, or for the
      // independent block-MSE rule the squared error of rounding the block's
      // values one by one (no in-block update, no curvature weight)
      double sel = 0.0;
      if constexpr (kRule == kRuleBlockMse) {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const double x = __dmul_rn(v[j], inv_s);
          const double r = e2m1_round_mag(fabs(x));
          const double res = __fma_rn(x < 0.0 ? r : -r, s, v[j]);
          sel = __fma_rn(res, res, sel);
        }
      }
      double dl[16];
      uint32_t sq[16];
      const double score = replay(v, s, inv_s, Ud, idb, dl, sq);
      if constexpr (kRule == kRuleSchurReplay) sel = score;

      // the chosen candidate: k0 for the amax rule, else the argmin of the
      // selection score over the 16 candidates, ties to the lower code
      int bl = k0 - lo;
      if constexpr (kRule != kRuleAmax) {
        double bs = sel;
        bl = hl;
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) {
          const double os = __shfl_xor_sync(FULL, bs, o, 16);
          const int ol = __shfl_xor_sync(FULL, bl, o, 16);
          if (os < bs || (os == bs && ol < bl)) {
            bs = os;
            bl = ol;
          }
        }
      }
      const double best = __shfl_sync(FULL, score, bl, 16);   // the winner's sum delta^2
      const bool live = amax > 0.0;
      __syncwarp();
      if (hl == bl) {
        // the winner publishes its deltas in place of the block's values and
        // its rounded magnitudes for the code nibbles
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          row[16 * b + j] = live ? dl[j] : 0.0;
          mrow[j] = sq[j];
        }
      }
      if (live) rowsum += best;
      __syncwarp();
      {
        // lane hl encodes column hl of the winner; the 16 nibbles are OR-ed
        // into the block's 8 code bytes (low nibble = even column)
        const uint32_t nib = live ? e2m1_nibble_hi(mrow[hl]) : 0u;
        uint32_t lo_w = hl < 8 ? nib << (4 * hl) : 0u, hi_w = hl < 8 ? 0u : nib << (4 * (hl - 8));
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) {
          lo_w |= __shfl_xor_sync(FULL, lo_w, o, 16);
          hi_w |= __shfl_xor_sync(FULL, hi_w, o, 16);
        }
        if (valid && hl == 0) {
          *reinterpret_cast<uint2*>(codes + r * (d_in / 2) + (c0 + 16 * b) / 2) =
              make_uint2(lo_w, hi_w);
          scales[r * (d_in / kBlock) + (c0 / kBlock) + b] = (uint8_t)(live ? lo + bl : 0);
        }
      }
      // later columns of the batch absorb the chosen block's deltas
      if (b + 1 < nblk) {
        double d[16];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const double2 dd = reinterpret_cast<const double2*>(row + 16 * b)[j];
          d[2 * j] = dd.x;
          d[2 * j + 1] = dd.y;
        }
        for (int q = b + 1; q < nblk; ++q) {
          const double* Uq = Ut + utile(b, q) * 256 + hl;
          double acc = row[16 * q + hl];
#pragma unroll
          for (int j = 0; j < 16; ++j) acc = __fma_rn(-d[j], Uq[16 * j], acc);
          row[16 * q + hl] = acc;
        }
      }
      __syncwarp();
    }
    if (valid) {
      for (int c = hl; c < bw; c += 16) {
        const double x = row[c];
        const float h = sm100::tf32_rn((float)x);
        Dh[r * ldD + kofs + c] = h;
        Dl[r * ldD + kofs + c] = (float)(x - (double)h);
      }
      if (hl == 0) rowerr[r] += rowsum;
    }
    __syncwarp();
  }
}

// One CTA per problem of the group: err = sum of its rows' delta^2.
__global__ void sum_rows_kernel(const QuantTable* __restrict__ tab,
                                const double* __restrict__ rowerr_all, int64_t n) {
  __shared__ double part[32];
  double* out = tab->err[blockIdx.x];
  if (!out) return;
  const double* rowerr = rowerr_all + (int64_t)blockIdx.x * n;
  double s = 0.0;
  for (int64_t i = threadIdx.x; i < n; i += blockDim.x) s += rowerr[i];
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x < 32) {
    s = (threadIdx.x < (blockDim.x >> 5)) ? part[threadIdx.x] : 0.0;
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (threadIdx.x == 0) *out = s;
  }
}

int grid_for(int64_t n, int threads) {
  int64_t b = (n + threads - 1) / threads;
  return (int)(b < 8 * kNumSMs ? (b < 1 ? 1 : b) : 8 * kNumSMs);
}

constexpr size_t kReplaySmem =
    sizeof(double) * (kUTiles * 256 + kLazyBatch + 2 * 128 + kRowsPerCta * kLazyBatch) +
    sizeof(uint32_t) * kRowsPerCta * 16;

}  // namespace

size_t quantize_ws_bytes(int64_t d_out, int64_t d_in) { return quant_group_bytes(d_out, d_in, 1); }
size_t quantize_group_ws_bytes(int64_t d_out, int64_t d_in, int P) {
  return quant_group_bytes(d_out, d_in, P);
}

const int* quantize_group_problem_status(const void* ws, int i) {
  const char* p = static_cast<const char*>(ws) + kWsHeader + align256(sizeof(QuantTable));
  return reinterpret_cast<const int*>(p + sizeof(QuantHeader) * i);
}

nvfp4_status launch_weight_amax(const void* W, nvfp4_dtype wt, int64_t d_out, int64_t d_in,
                                const uint8_t* dead, float* amax, cudaStream_t st) {
  NVFP4_CUDA_TRY(cudaMemsetAsync(amax, 0, sizeof(float), st));
  if (d_out == 0 || d_in == 0) return NVFP4_OK;
  const int g = grid_for(d_out * d_in, 256);
  unsigned* bits = reinterpret_cast<unsigned*>(amax);
  if (wt == NVFP4_BF16)
    weight_amax_kernel<uint16_t><<<g, 256, 0, st>>>(static_cast<const uint16_t*>(W), d_out,
                                                    d_in, dead, bits);
  else
    weight_amax_kernel<float><<<g, 256, 0, st>>>(static_cast<const float*>(W), d_out, d_in,
                                                 dead, bits);
  NVFP4_LAUNCH_CHECK();
  count_launches(1);
  return NVFP4_OK;
}

// GPTQ with Schur Replay for a group of P weight matrices of one shape (each
// with its own U, outputs and global scale; every launch covers all P): ws is
// the group region (quantize_group_ws_bytes(d_out, d_in, P) bytes).
nvfp4_status launch_quantize_group(int P, const PtrArr<const void*>& W, nvfp4_dtype wt,
                                   int64_t d_out, int64_t d_in, const PtrArr<const float*>& U,
                                   const PtrArr<const uint8_t*>& dead, int rule,
                                   const PtrArr<uint8_t*>& codes, const PtrArr<uint8_t*>& scales,
                                   const PtrArr<float*>& sg, const PtrArr<double*>& err,
                                   const PtrArr<const float*>& amax_in, void* ws,
                                   cudaStream_t st) {
  if (P < 1 || P > kMaxGroup) return NVFP4_ERR_INVALID_ARG;
  QuantLayout L = quant_layout(ws, d_out, d_in, P);
  {
    QuantTable t;
    for (int i = 0; i < P; ++i) {
      t.W[i] = W.p[i];
      t.U[i] = U.p[i];
      t.dead[i] = dead.p[i];
      t.codes[i] = codes.p[i];
      t.scales[i] = scales.p[i];
      t.sg[i] = sg.p[i];
      t.err[i] = err.p[i];
      t.amax_in[i] = amax_in.p[i];
    }
    for (int i = P; i < kMaxGroup; ++i) {
      t.W[i] = t.U[i] = nullptr;
      t.dead[i] = nullptr;
      t.codes[i] = t.scales[i] = nullptr;
      t.sg[i] = nullptr;
      t.err[i] = nullptr;
      t.amax_in[i] = nullptr;
    }
    init_group_kernel<<<1, 256, 0, st>>>(t, L.tab, L.gstatus, L.hdr, P);
    NVFP4_LAUNCH_CHECK();
    count_launches(1);
  }
  if (d_out == 0 || d_in == 0) {
    global_scale_kernel<<<1, kMaxGroup, 0, st>>>(L.tab, L.hdr, P);
    NVFP4_LAUNCH_CHECK();
    count_launches(1);
    for (int i = 0; i < P; ++i)
      if (err.p[i]) NVFP4_CUDA_TRY(cudaMemsetAsync(err.p[i], 0, sizeof(double), st));
    return NVFP4_OK;
  }
  {
    int g = grid_for(d_out * d_in / 8, 256) / P;
    g = g < 1 ? 1 : g;
    const dim3 wg((unsigned)g, (unsigned)P);
    if (wt == NVFP4_BF16)
      wprep_kernel<uint16_t><<<wg, 256, 0, st>>>(L.tab, d_out, d_in, L.Wt, L.rowerr, L.hdr,
                                                 L.gstatus);
    else
      wprep_kernel<float><<<wg, 256, 0, st>>>(L.tab, d_out, d_in, L.Wt, L.rowerr, L.hdr,
                                              L.gstatus);
    NVFP4_LAUNCH_CHECK();
    global_scale_kernel<<<1, kMaxGroup, 0, st>>>(L.tab, L.hdr, P);
    NVFP4_LAUNCH_CHECK();
    count_launches(2);
  }

  auto* replay_kernel = rule == kRuleAmax       ? schur_replay_batch_kernel<kRuleAmax>
                       : rule == kRuleBlockMse ? schur_replay_batch_kernel<kRuleBlockMse>
                                               : schur_replay_batch_kernel<kRuleSchurReplay>;
  NVFP4_CUDA_TRY(cudaFuncSetAttribute(replay_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)kReplaySmem));
  UpdateMaps maps;
  if (!make_update_maps(&maps, L.Dh, L.Dl, L.Uh, L.Ul, L.Wt, d_out, d_in, L.S, P))
    return NVFP4_ERR_CUDA;
  // CTAs per problem: one CTA per SM for a single problem; for a group,
  // enough CTAs of about 8 row groups each that the tail of the last wave is
  // a small part of the launch (each CTA stages its problem's U tiles once)
  const int64_t rg = (d_out + kRowsPerCta - 1) / kRowsPerCta;
  int64_t want = (rg * P + 7) / 8;
  if (want < kNumSMs) want = kNumSMs;
  int64_t per_problem = (want + P - 1) / P;
  if (per_problem > rg) per_problem = rg;
  const dim3 rgrid((unsigned)per_problem, (unsigned)P);
  const int64_t sW = d_out * d_in, sD = d_out * L.S, sU = d_in * L.S;
  for (int64_t cs = 0; cs < d_in; cs += L.S) {
    const int64_t send = (d_in - cs) < L.S ? d_in : cs + L.S;
    const int64_t j0 = cs + kLazyBatch;   // first column any update of this super-batch touches
    if (j0 < d_in) {
      ProfileScope ps(kPhaseUpdate, st);
      const int nk = (int)(send - cs);
      NVFP4_CUDA_TRY(launch_chained(split_u_rows_kernel,
                                    dim3((unsigned)((d_in - j0 + 31) / 32),
                                         (unsigned)((nk + 31) / 32), (unsigned)P),
                                    dim3(256), 0, st, (const QuantTable*)L.tab, (int64_t)d_in,
                                    cs, nk, j0, L.S, L.Uh, L.Ul));
      count_launches(1);
    }
    for (int64_t c0 = cs; c0 < send; c0 += kLazyBatch) {
      const int bw = (int)((d_in - c0) < kLazyBatch ? (d_in - c0) : kLazyBatch);
      const int kofs = (int)(c0 - cs);
      {
        ProfileScope ps(kPhaseReplay, st);
        NVFP4_CUDA_TRY(launch_chained(replay_kernel, rgrid, dim3(kReplayThreads),
                                      kReplaySmem, st, (const QuantTable*)L.tab, L.Wt, d_out,
                                      d_in, (int)c0, bw, L.Dh, L.Dl, L.S, kofs, L.rowerr));
        count_launches(1);
      }
      const int64_t e = c0 + bw;
      if (e < send) {
        // the batch's deltas into the rest of the super-batch (W~ slab kept in L2)
        ProfileScope ps(kPhaseUpdate, st);
        nvfp4_status s = launch_update_tc(maps, d_out, d_in, e, send, kofs, 1, true, P,
                                          L.gstatus, st);
        if (s != NVFP4_OK) return s;
      }
    }
    if (send < d_in) {
      // the whole super-batch's deltas into every later column, K = send - cs:
      // the 3xTF32 GEMM engine on the deltas' and U's hi/lo parts (128 x 128
      // tiles, 128-deep partials summed in fp32 registers), added to the fp64
      // working copy in its epilogue; one batch entry per problem
      ProfileScope ps(kPhaseUpdate, st);
      nvfp4_status s = gemm_nt_tc_split(
          (int)d_out, (int)(d_in - send), (int)(send - cs), -1.f, L.Dh, L.Dl, L.S, sD,
          L.Uh + send * L.S, L.Ul + send * L.S, L.S, sU, 0.f, nullptr, d_in, sW, nullptr, 0, 0,
          P, 0, L.gstatus, st, L.Wt + send);
      if (s != NVFP4_OK) return s;
    }
  }
  sum_rows_kernel<<<P, 1024, 0, st>>>(L.tab, L.rowerr, d_out);
  NVFP4_LAUNCH_CHECK();
  count_launches(1);
  return NVFP4_OK;
}

// The single-problem quantize: a group of one whose region is ws.
nvfp4_status launch_quantize(const void* W, nvfp4_dtype wt, int64_t d_out, int64_t d_in,
                             const float* U, const uint8_t* dead, int rule, uint8_t* codes,
                             uint8_t* scales, float* sg, double* err, void* ws,
                             cudaStream_t st, const float* amax_in) {
  PtrArr<const void*> w;
  PtrArr<const float*> u, am;
  PtrArr<const uint8_t*> dd;
  PtrArr<uint8_t*> c, sc;
  PtrArr<float*> g;
  PtrArr<double*> e;
  w.p[0] = W;
  u.p[0] = U;
  dd.p[0] = dead;
  c.p[0] = codes;
  sc.p[0] = scales;
  g.p[0] = sg;
  e.p[0] = err;
  am.p[0] = amax_in;
  return launch_quantize_group(1, w, wt, d_out, d_in, u, dd, rule, c, sc, g, e, am, ws, st);
}

}  // namespace nvfp4

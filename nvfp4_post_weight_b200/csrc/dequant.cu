// a9: dequantization Q = e2m1(code) * e4m3(scale) * s_g, and a10: the layer
// error tr((W - Q) H (W - Q)^T).
//
// "Replay the Curvature", Abstract: every 16 E2M1 weights share one E4M3 block
// scale; the per-tensor fp32 global scale s_g multiplies both.  e2m1 * e4m3 has
// at most 6 significant bits and is exact in fp32, so the fp32 result
// (e2m1 * e4m3) * s_g is the correctly rounded full product.  For bf16 output
// the product is formed with round-to-odd in fp32 (round toward zero, then the
// sticky bit from the exact residual) and then rounded to bf16, which is again
// the correctly rounded full product (24 >= 8 + 2 bits).
#include <cuda_bf16.h>

#include "common.cuh"
#include "sm100.cuh"
#include "nvfp4_format.cuh"

namespace nvfp4 {
namespace {

__device__ __forceinline__ uint16_t bf16_of_product(float cs, float sg) {
  float hi = __fmul_rz(cs, sg);
  const float lo = fmaf(cs, sg, -hi);  // exact residual (normal products)
  if (lo != 0.f) hi = __uint_as_float(__float_as_uint(hi) | 1u);
  return __bfloat16_as_ushort(__float2bfloat16_rn(hi));
}

// bf16 bits of p, an exact product (cs * sg: 6 + 24 significant bits, exact in
// fp64), rounded once to nearest-even on bf16's grid: spacing 2^(e - 7) in
// the binade 2^e, 2^-133 below the normal range, overflow to infinity.  Used
// for products outside the normal fp32 range, where the fp32 residual of
// bf16_of_product is no longer exact.
__device__ __forceinline__ uint16_t bf16_of_exact(double p) {
  const double a = fabs(p);
  const uint32_t sign = (uint32_t)(__double2hiint(p) >> 31) << 15;
  if (a == 0.0) return (uint16_t)sign;
  int e = ilogb(a);
  e = e < -126 ? -126 : e;
  const double M = scalbn(1.5, e + 45);          // unit in the last place 2^(e - 7)
  const float r = (float)__dsub_rn(__dadd_rn(a, M), M);   // on bf16's grid: exact (or inf)
  return (uint16_t)((__float_as_uint(r) >> 16) | sign);
}

// The 16 dequantized values of one block: code bytes c (low nibble first),
// scale code sc, written to o (16 bf16 = 32 bytes, or 16 fp32 = 64 bytes),
// one product and one rounding per element.
template <bool kBF16>
__device__ __forceinline__ void dequant_block_exact(uint2 c, uint32_t sc, float sg, void* o) {
  const float sb = (float)e4m3_value(sc & 0x7F);
  const uint64_t p = ((uint64_t)c.y << 32) | c.x;
  float cs[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) cs[j] = e2m1_value((uint32_t)(p >> (4 * j)) & 0xF) * sb;
  if constexpr (kBF16) {
    uint32_t h[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
      h[j] = (uint32_t)bf16_of_exact((double)cs[2 * j] * (double)sg) |
             ((uint32_t)bf16_of_exact((double)cs[2 * j + 1] * (double)sg) << 16);
    uint4* q = reinterpret_cast<uint4*>(o);
    q[0] = make_uint4(h[0], h[1], h[2], h[3]);
    q[1] = make_uint4(h[4], h[5], h[6], h[7]);
  } else {
    float4* q = reinterpret_cast<float4*>(o);
#pragma unroll
    for (int k = 0; k < 4; ++k)
      q[k] = make_float4(cs[4 * k] * sg, cs[4 * k + 1] * sg, cs[4 * k + 2] * sg,
                         cs[4 * k + 3] * sg);
  }
}

// bf16 output by table.  An E2M1 magnitude is 1 or 3 times a power of two
// (0.5, 1, 2, 4 and 1.5, 3, 6), so every element of a block is
// 2^k bf16(sb sg) or 2^k bf16(3 sb sg): the block takes two correctly rounded
// products, and scaling a normal bf16 by 2^k is exact (an add to its exponent
// field).  The eight magnitudes' bf16 bits form a table whose low and high
// bytes sit in two register pairs; one byte permutation per register pair
// looks up four elements at once (selector = the 3-bit magnitudes), a third
// interleaves low and high bytes, and the sign bits come from the code bits
// by a fourth.  Blocks whose products come near either end of the normal
// range take the exact path; a scale code of 0 gives a table of zeros.
__device__ __forceinline__ void dequant_block_bf16(uint2 c, uint32_t sc, float sg, void* o) {
  const uint32_t s7 = sc & 0x7F;
  // e4m3 value: (8 + m) 2^(e - 10) for e >= 1 (as fp32 bits), m 2^-9 for e == 0
  const float sb =
      (s7 & 0x78) ? __uint_as_float((s7 << 20) + 0x3C000000u) : (float)s7 * 0x1p-9f;
  const uint32_t b1 = bf16_of_product(sb, sg), b3 = bf16_of_product(3.f * sb, sg);
  const uint32_t e1 = (b1 >> 7) & 0xFF, e3 = (b3 >> 7) & 0xFF;
  // b1 and b3 are exact through the fp32 residual while every bit of the
  // product is at or above 2^-149 (products from 2^-118 up: e1 >= 10), and
  // 2^-1 b1 ... 2 b3 stay normal and finite for e1 >= 10, e3 <= 252
  if (s7 != 0 && (e1 < 10 || e3 > 252)) {
    dequant_block_exact<true>(c, sc, sg, o);
    return;
  }
  const uint32_t z = s7 ? 0xFFFFFFFFu : 0u;
  // magnitudes 0, 1/2, 1, 3/2 | 2, 3, 4, 6 as bf16 bits, two per word
  const uint32_t t01 = ((b1 - 0x80u) << 16) & z;
  const uint32_t t23 = (b1 | ((b3 - 0x80u) << 16)) & z;
  const uint32_t t45 = ((b1 + 0x80u) | (b3 << 16)) & z;
  const uint32_t t67 = ((b1 + 0x100u) | ((b3 + 0x80u) << 16)) & z;
  const uint32_t L0 = __byte_perm(t01, t23, 0x6420), H0 = __byte_perm(t01, t23, 0x7531);
  const uint32_t L1 = __byte_perm(t45, t67, 0x6420), H1 = __byte_perm(t45, t67, 0x7531);
  uint32_t h[8];
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const uint32_t w = q ? c.y : c.x;   // eight code nibbles
    const uint32_t m0 = w & 0x7777u, m1 = (w >> 16) & 0x7777u;
    const uint32_t l0 = __byte_perm(L0, L1, m0), h0 = __byte_perm(H0, H1, m0);
    const uint32_t l1 = __byte_perm(L0, L1, m1), h1 = __byte_perm(H0, H1, m1);
    // byte k of s4 / s8 carries the sign of element 2k / 2k + 1 in its top bit
    const uint32_t s4 = (w << 4) & 0x80808080u, s8 = w & 0x80808080u;
    h[4 * q + 0] = __byte_perm(l0, h0, 0x5140) | (__byte_perm(s4, s8, 0x4400) & 0x80008000u);
    h[4 * q + 1] = __byte_perm(l0, h0, 0x7362) | (__byte_perm(s4, s8, 0x5511) & 0x80008000u);
    h[4 * q + 2] = __byte_perm(l1, h1, 0x5140) | (__byte_perm(s4, s8, 0x6622) & 0x80008000u);
    h[4 * q + 3] = __byte_perm(l1, h1, 0x7362) | (__byte_perm(s4, s8, 0x7733) & 0x80008000u);
  }
  uint4* d = reinterpret_cast<uint4*>(o);
  d[0] = make_uint4(h[0], h[1], h[2], h[3]);
  d[1] = make_uint4(h[4], h[5], h[6], h[7]);
}

template <bool kBF16>
__device__ __forceinline__ void dequant_block(uint2 c, uint32_t sc, float sg, void* o) {
  if constexpr (kBF16)
    dequant_block_bf16(c, sc, sg, o);
  else
    dequant_block_exact<false>(c, sc, sg, o);
}

// Problem blockIdx.y of a group.  Each thread step takes four 16-weight blocks
// one grid stride apart (so that every load instruction of a warp reads 32
// consecutive blocks' bytes), all loads issued before any use; the output of
// a warp's blocks is one contiguous run per store pair.
template <bool kBF16>
__global__ void dequant_kernel(PtrArr<const uint8_t*> codes_a, PtrArr<const uint8_t*> scales_a,
                               PtrArr<const float*> sg_a, PtrArr<void*> out_a,
                               int64_t nblocks) {
  const int pb = blockIdx.y;
  const uint2* __restrict__ codes = reinterpret_cast<const uint2*>(codes_a.p[pb]);
  const uint8_t* __restrict__ scales = scales_a.p[pb];
  uint8_t* out = static_cast<uint8_t*>(out_a.p[pb]);
  constexpr int kOut = kBF16 ? 32 : 64;   // output bytes per block
  const float sg = *sg_a.p[pb];
  const int64_t T = (int64_t)gridDim.x * blockDim.x;
  const int64_t t0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  int64_t b = t0;
  for (; b + 3 * T < nblocks; b += 4 * T) {
    uint2 c[4];
    uint32_t sc[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) c[k] = codes[b + k * T];
#pragma unroll
    for (int k = 0; k < 4; ++k) sc[k] = scales[b + k * T];
#pragma unroll
    for (int k = 0; k < 4; ++k) dequant_block<kBF16>(c[k], sc[k], sg, out + (b + k * T) * kOut);
  }
  for (; b < nblocks; b += T) dequant_block<kBF16>(codes[b], scales[b], sg, out + b * kOut);
}

// Et = (W - Q)^T in fp32 (W bf16 or fp32) for a 64 x 64 tile of W: one
// thread per (row, 16-weight block) computes its 16 errors with a single
// rounding each, the tile is transposed through shared memory, and Et's rows
// (ldE >= d_out apart) are written whole -- already split for the 3xTF32
// Gram product: Eh = tf32(Et), El = Et - Eh (exact).
// Problem blockIdx.z of a group: its Eh/El a whole ldE x d_in array after the
// previous problem's.
template <typename T>
__global__ void __launch_bounds__(256)
    error_t_kernel(PtrArr<const void*> Ws, PtrArr<const uint8_t*> codes_a,
                   PtrArr<const uint8_t*> scales_a, PtrArr<const float*> sg_a, int64_t d_out,
                   int64_t d_in, float* __restrict__ Eh, float* __restrict__ El, int64_t ldE) {
  __shared__ float tile[64][65];
  const int pb = blockIdx.z;
  const T* __restrict__ W = static_cast<const T*>(Ws.p[pb]);
  const uint8_t* __restrict__ codes = codes_a.p[pb];
  const uint8_t* __restrict__ scales = scales_a.p[pb];
  Eh += (int64_t)pb * ldE * d_in;
  El += (int64_t)pb * ldE * d_in;
  const float sg = *sg_a.p[pb];
  const int64_t r0 = (int64_t)blockIdx.y * 64, c0 = (int64_t)blockIdx.x * 64;
  const int t = threadIdx.x, row = t >> 2, blk = t & 3;
  const int64_t r = r0 + row, cb = c0 + 16 * blk;
  if (r < d_out && cb < d_in) {
    const int64_t b = r * (d_in / 16) + cb / 16;
    const uint2 c = reinterpret_cast<const uint2*>(codes)[b];
    const float sb = (float)e4m3_value(scales[b] & 0x7F);
    const uint64_t p = ((uint64_t)c.y << 32) | c.x;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      float w;
      if constexpr (sizeof(T) == 2)
        w = __uint_as_float((uint32_t)W[r * d_in + cb + j] << 16);
      else
        w = W[r * d_in + cb + j];
      // w - (e2m1 * e4m3) * s_g with a single rounding
      tile[16 * blk + j][row] = fmaf(-e2m1_value((uint32_t)(p >> (4 * j)) & 0xF) * sb, sg, w);
    }
  } else {
#pragma unroll
    for (int j = 0; j < 16; ++j) tile[16 * blk + j][row] = 0.f;
  }
  __syncthreads();
#pragma unroll
  for (int q = 0; q < 16; ++q) {
    const int idx = t + 256 * q, j = idx >> 6, rr = idx & 63;
    if (c0 + j < d_in && r0 + rr < d_out) {
      const float v = tile[j][rr], h = sm100::tf32_rn(v);
      Eh[(c0 + j) * ldE + r0 + rr] = h;
      El[(c0 + j) * ldE + r0 + rr] = v - h;
    }
  }
}

// sum_ij H_ij G_ij in fp64 with G = E^T E known on the 128 x 128 tiles on or
// below the diagonal only (the tile size of gemm_nt_tc's lower mode): by the
// symmetry of G and H an off-diagonal tile stands for its mirror image too
// (weight 2), a diagonal tile for itself.  Rows are shared out over the CTAs;
// tiles above the diagonal are not read.  Four consecutive columns per thread
// and step (d and the tile edges are multiples of 4), read as float4 when H
// is 16-byte aligned (vec; G is workspace), so that several loads are in
// flight per thread.
// Problem blockIdx.y of a group: its G a d x d array after the previous
// problem's, its partial sums gridDim.x doubles after.
__global__ void sym_tile_dot_kernel(PtrArr<const float*> Hs, const float* __restrict__ G,
                                    int64_t d, double* __restrict__ partial) {
  __shared__ double part[32];
  const int pb = blockIdx.y;
  const float* __restrict__ H = Hs.p[pb];
  G += (int64_t)pb * d * d;
  partial += (int64_t)pb * gridDim.x;
  const bool vec = (reinterpret_cast<uintptr_t>(H) & 15) == 0;
  double s = 0.0;
  for (int64_t i = blockIdx.x; i < d; i += gridDim.x) {
    const int64_t jdiag = (i / 128) * 128;
    const int64_t jend = (jdiag + 128) < d ? (jdiag + 128) : d;
    const float* hr = H + i * d;
    const float* gr = G + i * d;
#pragma unroll 2
    for (int64_t j = 4 * (int64_t)threadIdx.x; j < jend; j += 4 * (int64_t)blockDim.x) {
      float4 h;
      if (vec) {
        h = *reinterpret_cast<const float4*>(hr + j);
      } else {
        h = make_float4(hr[j], hr[j + 1], hr[j + 2], hr[j + 3]);
      }
      const float4 g = *reinterpret_cast<const float4*>(gr + j);
      const double t = (double)h.x * (double)g.x + (double)h.y * (double)g.y +
                       (double)h.z * (double)g.z + (double)h.w * (double)g.w;
      s += j < jdiag ? 2.0 * t : t;   // the four share a side: jdiag is a multiple of 4
    }
  }
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x < 32) {
    s = (threadIdx.x < (blockDim.x >> 5)) ? part[threadIdx.x] : 0.0;
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (threadIdx.x == 0) partial[blockIdx.x] = s;
  }
}

// The partial sums added by one warp in a fixed order (deterministic); one
// CTA per problem of a group.
__global__ void sum_partials_kernel(const double* __restrict__ p, int n, PtrArr<double*> outs) {
  double* out = outs.p[blockIdx.x];
  p += (int64_t)blockIdx.x * n;
  double s = 0.0;
  for (int i = threadIdx.x; i < n; i += 32) s += p[i];
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (threadIdx.x == 0) *out = s;
}

// Export of the block scales into 128-row x 4-column tiles of 512 bytes (the
// scale-operand layout of block-scaled tensor-core FP4 GEMMs): one thread per
// output byte, so the writes are coalesced; padding rows and columns get code 0.
__global__ void scales_tiled_kernel(const uint8_t* __restrict__ scales, int64_t rows,
                                    int64_t nb, int64_t n_ct, int64_t total,
                                    uint8_t* __restrict__ out) {
  for (int64_t o = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; o < total;
       o += (int64_t)gridDim.x * blockDim.x) {
    const int64_t tile = o >> 9;
    const int in = (int)(o & 511);
    const int a = in >> 4, b = (in >> 2) & 3, c = in & 3;   // byte 16 a + 4 b + c
    const int64_t r = (tile / n_ct) * 128 + 32 * b + a;
    const int64_t col = (tile % n_ct) * 4 + c;
    out[o] = (r < rows && col < nb) ? scales[r * nb + col] : (uint8_t)0;
  }
}

int grid_for(int64_t n, int threads) {
  int64_t b = (n + threads - 1) / threads;
  return (int)(b < 8 * kNumSMs ? (b < 1 ? 1 : b) : 8 * kNumSMs);
}

constexpr int kDotBlocks = 8 * kNumSMs;

}  // namespace

// P problems of one shape (codes, scales, s_g and outputs per problem).
nvfp4_status launch_dequant_group(int P, const PtrArr<const uint8_t*>& codes,
                                  const PtrArr<const uint8_t*>& scales,
                                  const PtrArr<const float*>& sg, const PtrArr<void*>& out,
                                  int64_t d_out, int64_t d_in, nvfp4_dtype ot, cudaStream_t st) {
  const int64_t nb = d_out * (d_in / kBlock);
  if (nb == 0 || P < 1) return NVFP4_OK;
  // many resident CTAs: each thread keeps four blocks' loads in flight, and
  // the write-heavy stream wants every SM's load/store queues full
  int64_t g = ((nb + 3) / 4 + 255) / 256;
  if (g > 32 * kNumSMs) g = 32 * kNumSMs;
  g /= P;
  const dim3 grid((unsigned)(g < 1 ? 1 : g), (unsigned)P);
  if (ot == NVFP4_BF16)
    dequant_kernel<true><<<grid, 256, 0, st>>>(codes, scales, sg, out, nb);
  else
    dequant_kernel<false><<<grid, 256, 0, st>>>(codes, scales, sg, out, nb);
  NVFP4_LAUNCH_CHECK();
  count_launches(1);
  return NVFP4_OK;
}

nvfp4_status launch_dequant(const uint8_t* codes, const uint8_t* scales, const float* sg,
                            int64_t d_out, int64_t d_in, void* out, nvfp4_dtype ot,
                            cudaStream_t st) {
  PtrArr<const uint8_t*> c, s;
  PtrArr<const float*> g;
  PtrArr<void*> o;
  c.p[0] = codes;
  s.p[0] = scales;
  g.p[0] = sg;
  o.p[0] = out;
  return launch_dequant_group(1, c, s, g, o, d_out, d_in, ot, st);
}

int64_t et_ld(int64_t d_out) { return (d_out + 31) / 32 * 32; }

size_t scales_tiled_bytes(int64_t rows, int64_t d_in) {
  const int64_t nb = d_in / kBlock;
  return (size_t)((rows + 127) / 128 * 128) * (size_t)((nb + 3) / 4 * 4);
}

nvfp4_status launch_scales_tiled(const uint8_t* scales, int64_t rows, int64_t d_in,
                                 uint8_t* out, cudaStream_t st) {
  const int64_t nb = d_in / kBlock;
  const int64_t total = (int64_t)scales_tiled_bytes(rows, d_in);
  if (total == 0) return NVFP4_OK;
  scales_tiled_kernel<<<grid_for(total, 256), 256, 0, st>>>(scales, rows, nb, (nb + 3) / 4,
                                                           total, out);
  NVFP4_LAUNCH_CHECK();
  count_launches(1);
  return NVFP4_OK;
}

size_t layer_error_group_ws_bytes(int64_t d_out, int64_t d_in, int P) {
  return kWsHeader + 2 * align256(sizeof(float) * et_ld(d_out) * d_in * P) +
         align256(sizeof(float) * d_in * d_in * P) + align256(sizeof(double) * kDotBlocks * P);
}

size_t layer_error_ws_bytes(int64_t d_out, int64_t d_in) {
  return layer_error_group_ws_bytes(d_out, d_in, 1);
}

// tr(E H E^T) = <H, E^T E>: the Gram matrix G = E^T E is a symmetric
// product, so only its tiles on or below the diagonal are formed (half the
// flops of E H), on the tensor cores (3xTF32), then dotted with H.  For a
// group of P problems of one shape every launch covers all P (the GEMM a batch
// of P); ws is the group region, its first int the status word.
nvfp4_status launch_layer_error_group(int P, const PtrArr<const void*>& W, nvfp4_dtype wt,
                                      const PtrArr<const uint8_t*>& codes,
                                      const PtrArr<const uint8_t*>& scales,
                                      const PtrArr<const float*>& sg,
                                      const PtrArr<const float*>& H, int64_t d_out, int64_t d_in,
                                      const PtrArr<double*>& err, void* ws, cudaStream_t st) {
  if (P < 1 || P > kMaxGroup) return NVFP4_ERR_INVALID_ARG;
  int* status = static_cast<int*>(ws);
  NVFP4_CUDA_TRY(cudaMemsetAsync(status, 0, sizeof(int), st));
  if (d_out == 0 || d_in == 0) {
    for (int i = 0; i < P; ++i)
      NVFP4_CUDA_TRY(cudaMemsetAsync(err.p[i], 0, sizeof(double), st));
    return NVFP4_OK;
  }
  char* p = static_cast<char*>(ws) + kWsHeader;
  const int64_t ldE = et_ld(d_out);
  const size_t et_bytes = align256(sizeof(float) * ldE * d_in * P);
  float* Eh = reinterpret_cast<float*>(p);
  float* El = reinterpret_cast<float*>(p + et_bytes);
  float* G = reinterpret_cast<float*>(p + 2 * et_bytes);
  double* part =
      reinterpret_cast<double*>(p + 2 * et_bytes + align256(sizeof(float) * d_in * d_in * P));
  const dim3 tgrid((unsigned)((d_in + 63) / 64), (unsigned)((d_out + 63) / 64), (unsigned)P);
  if (wt == NVFP4_BF16)
    error_t_kernel<uint16_t><<<tgrid, 256, 0, st>>>(W, codes, scales, sg, d_out, d_in, Eh, El, ldE);
  else
    error_t_kernel<float><<<tgrid, 256, 0, st>>>(W, codes, scales, sg, d_out, d_in, Eh, El, ldE);
  NVFP4_LAUNCH_CHECK();
  count_launches(1);
  // G = Et Et^T (d_in x d_in, K = d_out), lower tiles only, one batch entry per problem
  nvfp4_status s = gemm_nt_tc_split((int)d_in, (int)d_in, (int)d_out, 1.f, Eh, El, ldE,
                                    ldE * d_in, Eh, El, ldE, ldE * d_in, 0.f, G, d_in, d_in * d_in,
                                    nullptr, 0, 0, P, 1, status, st);
  if (s != NVFP4_OK) return s;
  sym_tile_dot_kernel<<<dim3(kDotBlocks, P), 256, 0, st>>>(H, G, d_in, part);
  NVFP4_LAUNCH_CHECK();
  sum_partials_kernel<<<P, 32, 0, st>>>(part, kDotBlocks, err);
  NVFP4_LAUNCH_CHECK();
  count_launches(2);
  return NVFP4_OK;
}

nvfp4_status launch_layer_error(const void* W, nvfp4_dtype wt, const uint8_t* codes,
                                const uint8_t* scales, const float* sg, const float* H,
                                int64_t d_out, int64_t d_in, double* err, void* ws,
                                cudaStream_t st) {
  PtrArr<const void*> w;
  PtrArr<const uint8_t*> c, sc;
  PtrArr<const float*> g, h;
  PtrArr<double*> e;
  w.p[0] = W;
  c.p[0] = codes;
  sc.p[0] = scales;
  g.p[0] = sg;
  h.p[0] = H;
  e.p[0] = err;
  return launch_layer_error_group(1, w, wt, c, sc, g, h, d_out, d_in, e, ws, st);
}

}  // namespace nvfp4

// Shared host/device helpers of the NVFP4 GPTQ library (sm_100a).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "nvfp4pw.h"

namespace nvfp4 {

constexpr int kBlock = 16;        // weights per E4M3 block scale
constexpr int kCand = 16;         // candidate scales per block
constexpr int kLazyBatch = 128;   // columns per lazy batch
constexpr int kNumSMs = 148;      // B200

// Workspace header: the sticky device status word lives in the first 256 bytes.
constexpr size_t kWsHeader = 256;

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Records the first non-OK status in the sticky word (device side).
__device__ __forceinline__ void flag_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// ---- groups: several problems of one shape in every launch ------------------
// A group is P <= kMaxGroup problems of the same shape.  Its scratch lives in
// one region: a 256-byte group header whose first int is the group's sticky
// status word, per-problem headers, then every scratch array as P copies a
// uniform stride apart, so that one launch (grid dimension or GEMM batch)
// covers all P problems.  The single-problem calls are groups of one: their
// workspace is one group region, and its first int is the status word
// nvfp4_workspace_status() reads.  Caller-owned buffers reach the kernels as
// per-problem pointer arrays (kernel parameters, or a table in the region).
constexpr int kMaxGroup = 256;
template <typename T>
struct PtrArr {
  T p[kMaxGroup];
};

// Batched calls: one workspace for all problems -- a batch header (the first
// int: the first non-OK status of any problem; then one status word per
// problem in the caller's order), then one group region per run of problems
// of equal shape (problems grouped by shape in their order of appearance, at
// most kMaxGroup per group).
__host__ __device__ inline size_t batch_header_bytes(int count) {
  return align256(sizeof(int) * (1 + (size_t)count));
}
// Copies each group problem's status (its own word, else the group's word)
// into the batch header at the problem's index in the call: idx[i] for
// problem i of the group; per_problem_status[i] points at problem i's word.
nvfp4_status gather_group_status(int* batch_hdr, const int* group_status,
                                 const PtrArr<const int*>& per_problem_status,
                                 const PtrArr<int>& idx, int P, cudaStream_t st);

inline cudaStream_t as_cuda(nvfp4_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

// ---- launch accounting and optional per-phase event timing (runtime.cu) ----
enum Phase {
  kPhaseHessian = 0,
  kPhasePrepare = 1,
  kPhaseReplay = 2,
  kPhaseUpdate = 3,
  kPhaseDequant = 4,
  kPhaseOther = 5,
  kPhaseFactorGemm = 6,   // sub-phases of kPhasePrepare
  kPhasePanel = 7,
  kPhaseFactorI8 = 8,
  kNumPhases = 9
};
// While profiling is on, adds algorithmic work (flops) to the open phase.
void add_phase_work(double work);
// Adds n to the library's kernel-launch counter (and to the open phase's).
void count_launches(int n);
// While profiling is on, records a CUDA event pair around its lifetime on
// `st` and charges the launches counted meanwhile to `phase`.
struct ProfileScope {
  ProfileScope(int phase, cudaStream_t st);
  ~ProfileScope();
  int slot;
  int prev_phase;
  cudaStream_t st;
};

// Debug-build check (NVFP4_DEBUG): true when cond holds; otherwise records
// NVFP4_ERR_BOUNDS in *status (first error wins) and yields false, so that
// the caller skips the access.  In the release build it is the constant true.
#ifdef NVFP4_DEBUG
#define NVFP4_DCHECK(cond, status)                                                  \
  ((cond) ? true : (atomicCAS((status), 0, (int)NVFP4_ERR_BOUNDS), false))
#else
#define NVFP4_DCHECK(cond, status) true
#endif

#define NVFP4_LAUNCH_CHECK()                                   \
  do {                                                         \
    if (cudaPeekAtLastError() != cudaSuccess) {                \
      cudaGetLastError();                                      \
      return NVFP4_ERR_CUDA;                                   \
    }                                                          \
  } while (0)

#define NVFP4_CUDA_TRY(x)                                      \
  do {                                                         \
    if ((x) != cudaSuccess) {                                  \
      cudaGetLastError();                                      \
      return NVFP4_ERR_CUDA;                                   \
    }                                                          \
  } while (0)

// SM count of the current device (cached per device).
int num_sms();
// 2-D tiled TMA descriptor: dims[0] innermost (elements), strides[0] = bytes
// between rows, box in elements; out-of-range elements read as zero.
bool encode_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype,
                    const uint64_t dims[2], const uint64_t strides[1], const uint32_t box[2],
                    CUtensorMapSwizzle swizzle);
// rank-D version: dims[rank], strides[rank-1] (bytes), box[rank].
bool encode_tmap_nd(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, int rank,
                    const uint64_t* dims, const uint64_t* strides, const uint32_t* box,
                    CUtensorMapSwizzle swizzle);

// C = beta C + alpha P Q^T on the tensor cores (3xTF32).  P: M x K, Q: N x K,
// C: M x N, all fp32 row-major with leading dimensions ld* (multiples of 4)
// and, for batch > 1, element strides stride* between the batch's matrices.
// C2 (optional): C^T is also written there.  lower: only the 128 x 128 tiles
// on or below the diagonal (M == N).  C64 (optional, then C is not written and
// beta must be 0): an fp64 destination, C64 += alpha P Q^T, the fp32 product
// added in fp64.  A timed-out wait sets *status.
nvfp4_status gemm_nt_tc(int M, int N, int K, float alpha, const float* P, int64_t ldp,
                        int64_t strideP, const float* Q, int64_t ldq, int64_t strideQ,
                        float beta, float* C, int64_t ldc, int64_t strideC, float* C2,
                        int64_t ldc2, int64_t strideC2, int batch, int lower, int* status,
                        cudaStream_t st, double* C64 = nullptr);
// The same product with both operands given already split for 3xTF32:
// Ph = tf32(P) and Pl = P - Ph (likewise Qh, Ql), same layout and strides.
nvfp4_status gemm_nt_tc_split(int M, int N, int K, float alpha, const float* Ph,
                              const float* Pl, int64_t ldp, int64_t strideP, const float* Qh,
                              const float* Ql, int64_t ldq, int64_t strideQ, float beta,
                              float* C, int64_t ldc, int64_t strideC, float* C2, int64_t ldc2,
                              int64_t strideC2, int batch, int lower, int* status,
                              cudaStream_t st, double* C64 = nullptr);

// C = beta C + alpha P Q^T in fp64 on the tensor cores (mma.sync m8n8k4; same
// operand conventions as gemm_nt_tc; C2 = C^T needs beta == 0; lower: only
// tiles on or below the diagonal; ktri: 0 dense P, 1 P upper triangular, 2 P
// lower triangular -- the zero part of K is skipped).  P and Q go through TMA:
// 16-byte aligned, even leading dimensions and batch strides, K a multiple of
// 16.  A wait that runs out records NVFP4_ERR_TIMEOUT in *status.
// The same product as dgemm_nt, fp64-accurate through int8 slices on tcgen05
// (kind::i8): P and Q cut into 7 power-of-two-scaled 7-bit slices per row,
// slice products exact in int32 TMEM, levels combined in fp64.  scratch holds
// the slices: dgemm_i8_scratch_bytes(M, N, K, batch) bytes.  K < 65536, K a
// multiple of 16.  A wait that runs out records NVFP4_ERR_TIMEOUT in *status.
size_t dgemm_i8_scratch_bytes(int64_t M, int64_t N, int64_t K, int batch);
nvfp4_status dgemm_i8(int M, int N, int K, double alpha, const double* P, int64_t ldp,
                      int64_t strideP, const double* Q, int64_t ldq, int64_t strideQ,
                      double beta, double* C, int64_t ldc, int64_t strideC, double* C2,
                      int64_t ldc2, int64_t strideC2, int batch, int lower, int ktri,
                      void* scratch, size_t scratch_bytes, int* status, cudaStream_t st);
nvfp4_status dgemm_nt(int M, int N, int K, double alpha, const double* P, int64_t ldp,
                      int64_t strideP, const double* Q, int64_t ldq, int64_t strideQ,
                      double beta, double* C, int64_t ldc, int64_t strideC, double* C2,
                      int64_t ldc2, int64_t strideC2, int batch, int lower, int ktri,
                      int* status, cudaStream_t st);

// ---- kernel launchers implemented in the .cu files -------------------------
bool hessian_tc_supported(const float* H, const void* X, nvfp4_dtype xt, int64_t n_tok,
                          int64_t d);
size_t hessian_host_ws_bytes(int64_t d, int64_t chunk_tok, nvfp4_dtype xt);
nvfp4_status launch_hessian_host(float* H, const void* X_host, nvfp4_dtype xt, int64_t n_tok,
                                 int64_t d, int beta, int64_t chunk_tok, void* ws,
                                 cudaStream_t st);
nvfp4_status launch_hessian_tc(float* H, const void* X, int64_t n_tok, int64_t d, int beta,
                               cudaStream_t st);
// P problems of one dimension d, each hessian_tc_supported (ragged n_tok).
nvfp4_status launch_hessian_tc_group(int P, float* const* H, const void* const* X,
                                     const int64_t* n_tok, int64_t d, int beta,
                                     cudaStream_t st);
int hessian_tc_take_status(cudaStream_t st);

// TMA descriptors of the tensor-core trailing update: Delta = Dh + Dl
// (d_out x 128, fp32 each) and the split rows U = Uh + Ul of one batch,
// transposed (d_in x 128, fp32 each, rows >= e used).
struct UpdateMaps {
  CUtensorMap Dh, Dl, Uh, Ul, W;   // W: the fp64 working copy (d_out x d_in)
};
// Maps of the update operands: Dh/Dl (d_out x kcols) and Uh/Ul (d_in x kcols)
// hold deltas and U rows K-contiguous, kcols K values per row.
// P problems of a group: each array repeats P times, a whole matrix apart.
bool make_update_maps(UpdateMaps* m, const float* Dh, const float* Dl, const float* Uh,
                      const float* Ul, const double* Wt, int64_t d_out, int64_t d_in,
                      int64_t kcols, int P);
// W~[:, e:e_end] -= sum over nkb 128-deep K blocks from K offset kofs of
// (Dh + Dl)(Uh + Ul)^T (3xTF32, fp64 W~); keep_w keeps W~ in L2 (evict last)
// instead of streaming it.  A timed-out wait sets NVFP4_ERR_TIMEOUT in *status.
nvfp4_status launch_update_tc(const UpdateMaps& m, int64_t d_out, int64_t d_in, int64_t e,
                              int64_t e_end, int kofs, int nkb, bool keep_w, int P, int* status,
                              cudaStream_t st);
nvfp4_status launch_hessian(float* H, const void* X, nvfp4_dtype xt, int64_t n_tok,
                            int64_t d, int beta, cudaStream_t st);
// H: fp32 (h64 false) or fp64 (h64 true), d x d.
nvfp4_status launch_prepare(const void* H, bool h64, int64_t d, float damp, float* U,
                            uint8_t* dead, float* lambda_out, void* ws, cudaStream_t st);
size_t hessian_f64_ws_bytes(int64_t n_tok, int64_t d);
nvfp4_status launch_hessian_f64(double* H, const void* X, nvfp4_dtype xt, int64_t n_tok,
                                int64_t d, int beta, void* ws, cudaStream_t st);
size_t prepare_ws_bytes(int64_t d);
// Groups of P problems of one shape (kernels launched once for all P); ws is
// the group region of *_group_ws_bytes() bytes.
size_t prepare_group_ws_bytes(int64_t d, int P);
nvfp4_status launch_prepare_group(int P, const PtrArr<const void*>& H, bool h64, int64_t d,
                                  float damp, const PtrArr<float*>& U,
                                  const PtrArr<uint8_t*>& dead, const PtrArr<float*>& lambda_out,
                                  void* ws, cudaStream_t st);
const int* prepare_group_problem_status(const void* ws, int i);
size_t quantize_group_ws_bytes(int64_t d_out, int64_t d_in, int P);
nvfp4_status launch_quantize_group(int P, const PtrArr<const void*>& W, nvfp4_dtype wt,
                                   int64_t d_out, int64_t d_in, const PtrArr<const float*>& U,
                                   const PtrArr<const uint8_t*>& dead, int rule,
                                   const PtrArr<uint8_t*>& codes, const PtrArr<uint8_t*>& scales,
                                   const PtrArr<float*>& sg, const PtrArr<double*>& err,
                                   const PtrArr<const float*>& amax_in, void* ws,
                                   cudaStream_t st);
const int* quantize_group_problem_status(const void* ws, int i);
nvfp4_status launch_quantize(const void* W, nvfp4_dtype wt, int64_t d_out, int64_t d_in,
                             const float* U, const uint8_t* dead, int rule, uint8_t* codes,
                             uint8_t* scales, float* sg, double* err, void* ws,
                             cudaStream_t st, const float* amax_in = nullptr);
size_t scales_tiled_bytes(int64_t rows, int64_t d_in);
nvfp4_status launch_scales_tiled(const uint8_t* scales, int64_t rows, int64_t d_in,
                                 uint8_t* out, cudaStream_t st);
nvfp4_status launch_weight_amax(const void* W, nvfp4_dtype wt, int64_t d_out, int64_t d_in,
                                const uint8_t* dead, float* amax, cudaStream_t st);
size_t quantize_ws_bytes(int64_t d_out, int64_t d_in);
nvfp4_status launch_dequant(const uint8_t* codes, const uint8_t* scales, const float* sg,
                            int64_t d_out, int64_t d_in, void* out, nvfp4_dtype ot,
                            cudaStream_t st);
nvfp4_status launch_dequant_group(int P, const PtrArr<const uint8_t*>& codes,
                                  const PtrArr<const uint8_t*>& scales,
                                  const PtrArr<const float*>& sg, const PtrArr<void*>& out,
                                  int64_t d_out, int64_t d_in, nvfp4_dtype ot, cudaStream_t st);
nvfp4_status launch_layer_error(const void* W, nvfp4_dtype wt, const uint8_t* codes,
                                const uint8_t* scales, const float* sg, const float* H,
                                int64_t d_out, int64_t d_in, double* err, void* ws,
                                cudaStream_t st);
size_t layer_error_ws_bytes(int64_t d_out, int64_t d_in);
size_t layer_error_group_ws_bytes(int64_t d_out, int64_t d_in, int P);
nvfp4_status launch_layer_error_group(int P, const PtrArr<const void*>& W, nvfp4_dtype wt,
                                      const PtrArr<const uint8_t*>& codes,
                                      const PtrArr<const uint8_t*>& scales,
                                      const PtrArr<const float*>& sg,
                                      const PtrArr<const float*>& H, int64_t d_out, int64_t d_in,
                                      const PtrArr<double*>& err, void* ws, cudaStream_t st);

// Programmatic dependent launch.  The kernels of a serial chain (panel ->
// update -> panel, replay -> update -> replay) are launched with
// launch_chained() and call pdl_wait() before their first global memory
// access; it returns once the previous kernel of the stream has completed and
// its writes are visible.  The launch itself and the set-up before the wait
// (barrier init, tensor-map prefetch, TMEM allocation) overlap the previous
// kernel's completion.  No kernel triggers its dependents early: measured on
// the 4096-wide layer, CTAs of the next kernel parked beside a running panel
// or GEMM slowed it more than the earlier start gained.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_chained(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                  cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// D (8x8) += A (8x4) B (4x8) in fp64 on the tensor cores (warp-wide
// mma.sync m8n8k4; tcgen05 has no fp64 kind).  Fragments per lane:
// a = A[lane/4][lane%4], b = B[lane%4][lane/4], d = D[lane/4][2*(lane%4)+{0,1}].
__device__ __forceinline__ void dmma_m8n8k4(double& d0, double& d1, double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};"
               : "+d"(d0), "+d"(d1)
               : "d"(a), "d"(b));
}

}  // namespace nvfp4

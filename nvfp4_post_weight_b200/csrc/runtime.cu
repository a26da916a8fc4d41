// Launch accounting and optional per-phase CUDA-event timing.
//
// Every kernel launch of the library is counted (nvfp4_launch_count), so a
// caller can check how many of the library's kernels a piece of work ran.
// While profiling is on, each launcher's ProfileScope records a CUDA event
// pair on the launching stream; nvfp4_profile_end() waits for the events and
// returns, per phase, the summed device time and the number of launches.
// Every ProfileScope also opens an NVTX range named for its phase (always,
// profiling on or off), so a tool attached through NVTX sees the phases.
#include <cudaTypedefs.h>
#include <nvtx3/nvToolsExt.h>

#include <atomic>
#include <mutex>
#include <vector>

#include "common.cuh"

namespace nvfp4 {
namespace {

struct Record {
  int phase;
  cudaEvent_t a, b;
};

std::mutex g_mu;
std::atomic<long long> g_launches{0};
std::atomic<long long> g_phase_launches[kNumPhases];
std::atomic<bool> g_profiling{false};
std::vector<Record> g_records;
double g_phase_work[kNumPhases];
std::vector<cudaEvent_t> g_pool;
thread_local int t_phase = -1;

cudaEvent_t get_event() {
  if (!g_pool.empty()) {
    cudaEvent_t e = g_pool.back();
    g_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return e;
}

}  // namespace

void count_launches(int n) {
  g_launches.fetch_add(n, std::memory_order_relaxed);
  const int p = t_phase >= 0 ? t_phase : kPhaseOther;
  g_phase_launches[p].fetch_add(n, std::memory_order_relaxed);
}

// Setters of every device module's pipeline-wait limit (sm100.cuh), one per
// .cu file, registered while the library loads.
using WaitSetter = cudaError_t (*)(unsigned long long);
static std::vector<WaitSetter>& wait_setters() {
  static std::vector<WaitSetter> v;   // constructed on first use: load order safe
  return v;
}
static std::mutex& wait_setters_mu() {
  static std::mutex m;
  return m;
}

int register_wait_limit_setter(cudaError_t (*setter)(unsigned long long ns)) {
  std::lock_guard<std::mutex> lk(wait_setters_mu());
  wait_setters().push_back(setter);
  return (int)wait_setters().size();
}

void add_phase_work(double work) {
  if (!g_profiling.load(std::memory_order_relaxed)) return;
  const int p = t_phase >= 0 ? t_phase : kPhaseOther;
  std::lock_guard<std::mutex> lk(g_mu);
  g_phase_work[p] += work;
}

// NVTX range names of the phases (nvfp4_phase order); a tool that attaches
// through NVTX sees every call's phases on the host timeline, and without one
// a push or pop costs a pointer test.
static const char* const kPhaseRangeNames[] = {
    "nvfp4 hessian", "nvfp4 prepare", "nvfp4 replay", "nvfp4 update", "nvfp4 dequant",
    "nvfp4 other",   "nvfp4 factor fp64 gemm", "nvfp4 panel", "nvfp4 factor int8 gemm"};

ProfileScope::ProfileScope(int phase, cudaStream_t s) : slot(-1), prev_phase(t_phase), st(s) {
  t_phase = phase;
  nvtxRangePushA(phase >= 0 && phase < (int)(sizeof(kPhaseRangeNames) / sizeof(kPhaseRangeNames[0]))
                     ? kPhaseRangeNames[phase]
                     : "nvfp4");
  if (!g_profiling.load(std::memory_order_relaxed)) return;
  std::lock_guard<std::mutex> lk(g_mu);
  Record r{phase, get_event(), get_event()};
  if (!r.a || !r.b) return;
  if (cudaEventRecord(r.a, st) != cudaSuccess) {
    cudaGetLastError();
    return;
  }
  slot = (int)g_records.size();
  g_records.push_back(r);
}

ProfileScope::~ProfileScope() {
  nvtxRangePop();
  t_phase = prev_phase;
  if (slot < 0) return;
  std::lock_guard<std::mutex> lk(g_mu);
  if (slot < (int)g_records.size() && cudaEventRecord(g_records[slot].b, st) != cudaSuccess) {
    cudaGetLastError();
    g_records[slot].phase = -1;
  }
}

// ---- device properties and TMA descriptors ---------------------------------
int num_sms() {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return kNumSMs;
  }
  int n = cache[dev].load(std::memory_order_relaxed);
  if (n > 0) return n;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    n = kNumSMs;
  }
  cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

bool encode_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype,
                    const uint64_t dims[2], const uint64_t strides[1], const uint32_t box[2],
                    CUtensorMapSwizzle swizzle) {
  return encode_tmap_nd(map, base, dtype, 2, dims, strides, box, swizzle);
}

bool encode_tmap_nd(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, int rank,
                    const uint64_t* dims, const uint64_t* strides, const uint32_t* box,
                    CUtensorMapSwizzle swizzle) {
  // The driver entry point is looked up at run time, so the library itself does
  // not link against libcuda.
  static PFN_cuTensorMapEncodeTiled_v12000 encode = [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess) {
      cudaGetLastError();
      fn = nullptr;
    }
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }();
  if (!encode || rank < 1 || rank > 5) return false;
  cuuint64_t gd[5], gs[5];
  cuuint32_t bd[5], es[5];
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bd[i] = box[i];
    es[i] = 1;
    if (i + 1 < rank) gs[i] = strides[i];
  }
  return encode(map, dtype, (cuuint32_t)rank, const_cast<void*>(base), gd, gs, bd, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace nvfp4

using namespace nvfp4;

extern "C" {

long long nvfp4_launch_count(void) { return g_launches.load(); }

int nvfp4_debug_build(void) {
#ifdef NVFP4_DEBUG
  return 1;
#else
  return 0;
#endif
}

nvfp4_status nvfp4_set_wait_limit_ns(unsigned long long ns) {
  const unsigned long long v = ns == 0 ? 4000000000ull : ns;
  std::lock_guard<std::mutex> lk(wait_setters_mu());
  for (WaitSetter f : wait_setters()) {
    if (f(v) != cudaSuccess) {
      cudaGetLastError();
      return NVFP4_ERR_CUDA;
    }
  }
  return NVFP4_OK;
}

nvfp4_status nvfp4_profile_begin(void) {
  std::lock_guard<std::mutex> lk(g_mu);
  for (auto& r : g_records) {
    g_pool.push_back(r.a);
    g_pool.push_back(r.b);
  }
  g_records.clear();
  for (int p = 0; p < kNumPhases; ++p) {
    g_phase_launches[p].store(0);
    g_phase_work[p] = 0.0;
  }
  g_profiling.store(true);
  return NVFP4_OK;
}

nvfp4_status nvfp4_profile_end(double* ms, long long* launches, int n_phases) {
  if (n_phases < 0 || (n_phases > 0 && (!ms || !launches))) return NVFP4_ERR_INVALID_ARG;
  g_profiling.store(false);
  std::lock_guard<std::mutex> lk(g_mu);
  for (int p = 0; p < n_phases; ++p) {
    ms[p] = 0.0;
    launches[p] = p < kNumPhases ? g_phase_launches[p].load() : 0;
  }
  nvfp4_status st = NVFP4_OK;
  for (auto& r : g_records) {
    if (r.phase < 0) continue;
    if (cudaEventSynchronize(r.b) != cudaSuccess) {
      cudaGetLastError();
      st = NVFP4_ERR_CUDA;
      continue;
    }
    float t = 0.f;
    if (cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess) {
      cudaGetLastError();
      st = NVFP4_ERR_CUDA;
      continue;
    }
    if (r.phase < n_phases) ms[r.phase] += (double)t;
  }
  for (auto& r : g_records) {
    g_pool.push_back(r.a);
    g_pool.push_back(r.b);
  }
  g_records.clear();
  return st;
}

nvfp4_status nvfp4_profile_work(double* work, int n_phases) {
  if (n_phases < 0 || (n_phases > 0 && !work)) return NVFP4_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_mu);
  for (int p = 0; p < n_phases; ++p) work[p] = p < kNumPhases ? g_phase_work[p] : 0.0;
  return NVFP4_OK;
}

}  // extern "C"

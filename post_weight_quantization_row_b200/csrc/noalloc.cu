// mpq_stage_energy_noalloc: the energy stage with its scratch in a fixed,
// file-scope device array instead of plan workspace.
//
// Some callers cannot let a library allocate device memory on its own: a
// process whose framework allocator owns every byte of the GPU, a serving
// loop that must not stall on the device-wide synchronisation that
// cudaMalloc/cudaFree can imply, or code that runs under a strict memory
// budget fixed at start-up.  This entry point serves them: it writes its
// intermediates into `g_noalloc_scratch` below and calls no allocator.
#include <mutex>

#include "mpq_internal.cuh"

namespace mpq {
namespace {

// Every device that loads the library keeps this array until the process exits.
constexpr size_t NOALLOC_SCRATCH_BYTES = (size_t)MPQ_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[NOALLOC_SCRATCH_BYTES];

constexpr int MAX_DEVICES = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[MAX_DEVICES] = {};

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Device address of the scratch array for the current device.  The host-side
// symbol is only a stand-in, so the address is looked up once per device
// (with that device current) and cached.
mpq_status scratch_for_current_device(void** out) {
  int dev = -1;
  MPQ_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= MAX_DEVICES) return fail(MPQ_ERR_UNSUPPORTED, "device index out of range");
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(g_noalloc_scratch)");
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return MPQ_OK;
}

}  // namespace
}  // namespace mpq

using namespace mpq;

extern "C" mpq_status mpq_stage_energy_noalloc(mpq_plan_t p, const float* W, int64_t m,
                                               const float* scale, const float* offset,
                                               const uint16_t* idx, float* w_hat, float* energy,
                                               mpq_stream_t stream) {
  if (!p) return fail(MPQ_ERR_INVALID_ARG, "plan is NULL");
  if (m < 0 || (m > 0 && (!W || !scale || !offset || !idx || !energy)))
    return fail(MPQ_ERR_INVALID_ARG, "energy_noalloc: missing buffer");
  if (m == 0) return MPQ_OK;
  // m * per_row > the array size already means refusal; checking it by
  // division first keeps the byte counts below from wrapping for huge m
  const uint64_t per_row = 4ull * (uint64_t)p->n + 4ull * (uint64_t)p->r + 2ull * (uint64_t)p->B;
  if (m > MAX_ROWS || (uint64_t)m > NOALLOC_SCRATCH_BYTES / per_row)
    return fail(MPQ_ERR_INVALID_ARG,
                "energy_noalloc: m * (4n + 4r + 2B) bytes exceeds the static scratch of " +
                    std::to_string(NOALLOC_SCRATCH_BYTES) + " bytes; split the rows");
  const size_t e_bytes = align256((size_t)m * p->n * sizeof(float));
  const size_t p_bytes = align256((size_t)m * p->r * sizeof(float));
  const size_t i_bytes = align256((size_t)m * p->B * sizeof(uint16_t));
  if (e_bytes + p_bytes + i_bytes > NOALLOC_SCRATCH_BYTES)
    return fail(MPQ_ERR_INVALID_ARG,
                "energy_noalloc: m * (4n + 4r + 2B) bytes exceeds the static scratch of " +
                    std::to_string(NOALLOC_SCRATCH_BYTES) + " bytes; split the rows");
  int cur = -1;
  MPQ_CUDA(cudaGetDevice(&cur));
  if (cur != p->device) return fail(MPQ_ERR_INVALID_ARG, "energy_noalloc: make the plan's device current");
  void* base = nullptr;
  MPQ_TRY(scratch_for_current_device(&base));
  cudaStream_t st = (cudaStream_t)stream;
  unsigned char* b = static_cast<unsigned char*>(base);
  float* E = reinterpret_cast<float*>(b);
  float* P = reinterpret_cast<float*>(b + e_bytes);
  uint16_t* safe = reinterpret_cast<uint16_t*>(b + e_bytes + p_bytes);
  // every scratch byte used below is written before it is read
  MPQ_CUDA(cudaMemcpyAsync(safe, idx, sizeof(uint16_t) * m * p->B, cudaMemcpyDeviceToDevice, st));
  MPQ_TRY(launch_sanitize_idx(p, safe, m * p->B, st));
  MPQ_TRY(launch_residual(p, W, m, scale, offset, safe, E, w_hat, st));
  MPQ_TRY(gemm_nt_f32(E, p->n, p->Vt32, p->n, P, p->r, m, p->r, p->n, st, "gemm_energy"));
  return launch_energy_rows(p, m, P, energy, st);
}

// dbsa_gather_rope_attend_noalloc: the Stage-2 call for callers that cannot
// hand the library a workspace.
//
// Some callers cannot allocate device memory when they call in: code that
// runs inside another framework's fixed memory budget (every byte of the
// device already belongs to a pool it does not own), or a host thread that
// must not call cudaMalloc (it may synchronise the device and stall other
// streams).  This entry point takes no workspace.  Its scratch (status word,
// RoPE tables, gather plan and split partials) lives in one fixed array in
// the library's own device memory, which every GPU that loads the library
// holds until the process exits.  The call makes no allocating CUDA call:
// the plan goes up with one cudaMemcpyAsync from pageable host memory rather
// than through the page-locked staging ring of the other entry points.
#include <cstdio>
#include <mutex>

#include "dbsa_internal.h"

namespace {

// Scratch of the no-allocation Stage-2 entry point: 16 MiB per device.
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
__device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  In host code
// g_noalloc_scratch names a host-side stand-in, not device memory, so the
// address is looked up once per device, with that device current, and kept.
cudaError_t scratch_for_current_device(void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" dbsa_status dbsa_gather_rope_attend_noalloc(
    const dbsa_config *cfg, const void *k_cache, const void *v_cache, int64_t cap,
    const int32_t *offs_host, int32_t nb, int32_t nq, const int32_t *sel_ptr_host,
    const int32_t *sel_blocks_host, const void *q_new, int32_t n_new, const void *k_tail,
    const void *v_tail, int32_t tail_len, int32_t tail_cap, void *out, int32_t *dbg_map,
    int64_t dbg_cap, void *stream) {
  // Validation and planning come first (a batch that needs more than the
  // array is rejected there, naming both sizes); the array's address is
  // looked up after that.  The call clears the status word at the head of the
  // scratch on `stream` before its kernels run and rewrites every other byte
  // it reads; the array keeps whatever the previous call left.
  const dbsa::FixedScratch fixed{kNoAllocScratchBytes, scratch_for_current_device};
  return dbsa::gather_fixed_scratch(cfg, k_cache, v_cache, cap, offs_host, nb, nq, sel_ptr_host,
                                    sel_blocks_host, q_new, n_new, k_tail, v_tail, tail_len,
                                    tail_cap, out, dbg_map, dbg_cap, fixed, stream);
}

extern "C" dbsa_status dbsa_noalloc_read_status(void *stream) {
  void *ws = nullptr;
  cudaError_t e = scratch_for_current_device(&ws);
  int word = 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (e == cudaSuccess) e = cudaMemcpyAsync(&word, ws, sizeof word, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) {
    char buf[256];
    snprintf(buf, sizeof buf, "dbsa_noalloc_read_status: %s", cudaGetErrorString(e));
    dbsa::set_last_error(buf);
    return DBSA_ERR_CUDA;
  }
  if (word == DBSA_ERR_TIMEOUT) dbsa::set_last_error("a device-side wait expired");
  return word == 0 ? DBSA_OK : static_cast<dbsa_status>(word);
}

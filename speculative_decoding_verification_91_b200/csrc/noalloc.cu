// LM head + argmax for callers that cannot allocate device memory.
//
// spec_lmhead_argmax needs a caller-provided workspace for its per-row argmax
// keys, its completion counter and its status word.  Some callers have no way
// to provide one: code that runs where device allocation is not permitted or
// not wanted (an inference runtime whose memory plan is fixed before the
// first token and forbids allocations on the decode path, a plugin handed
// only its input and output tensors by a host framework that owns every
// allocation, a latency-critical loop that cannot afford cudaMalloc's
// implicit device synchronisation).  spec_lmhead_argmax_noalloc serves them:
// its scratch is a file-scope __device__ array below, loaded with the
// library, so the call itself allocates nothing.
//
// Layout of the array: the 4 KiB header of every workspace (status word,
// then the completion counters), then one 64-bit argmax key per row.
#include <mutex>

#include "../../include/specverify.h"
#include "common.cuh"
#include "internal.h"

namespace sv {
namespace {

constexpr size_t kNoAllocHeader = kWsHeaderBytes;                       // status + counters
constexpr size_t kNoAllocEntries = (size_t)SPEC_NOALLOC_MAX_ROWS;       // argmax keys (one per row)
constexpr size_t kNoAllocBytes = kNoAllocHeader + kNoAllocEntries * 8;
// the status word is the header's first 4 bytes; counters start at word kTicketBase
constexpr size_t kNoAllocClearFrom = (size_t)kTicketBase * 4;

// One copy per GPU that loads the library; it stays allocated until exit.
__device__ __align__(256) uint8_t g_lmhead_scratch[kNoAllocBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  In host code
// `g_lmhead_scratch` names a host-side stand-in, not device memory, so the
// address must come from cudaGetSymbolAddress, once per device, with that
// device current.
int scratch_for_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SPEC_ECUDA;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_lmhead_scratch) != cudaSuccess || !p) return SPEC_ECUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return SPEC_OK;
}

// Host-side fault injection: OR bits into the status word (one thread).
__global__ void noalloc_inject_kernel(unsigned* status, unsigned bits) {
  pdl_trigger();
  pdl_wait();
  atomicOr(status, bits);
}

}  // namespace
}  // namespace sv

using namespace sv;

extern "C" int spec_lmhead_argmax_noalloc(const void* h, const void* w, int M, int d, int V,
                                          int32_t* ids, float* maxlogit, void* stream) {
  if (!h || !w || !ids || M < 1 || V < 1 || d < 8 || d % 8) return SPEC_EINVAL;
  if ((reinterpret_cast<uintptr_t>(h) & 15) || (reinterpret_cast<uintptr_t>(w) & 15)) return SPEC_EINVAL;
  // the fixed scratch holds one argmax key per row
  if (M > SPEC_NOALLOC_MAX_ROWS) return SPEC_EUNSUPPORTED;
  GemmPlan p = plan_gemm(M, V, d, kGemmArgmax);
  void* scratch = nullptr;
  int rc = scratch_for_current_device(&scratch);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // The array keeps the previous call's contents: the completion counters and
  // the argmax keys must start at zero (a call cut short by a timed-out wait
  // may have left them set).  The status word is kept: its bits accumulate
  // until spec_noalloc_read_status reads and clears them.
  if (cudaMemsetAsync(static_cast<uint8_t*>(scratch) + kNoAllocClearFrom, 0,
                      kNoAllocBytes - kNoAllocClearFrom, st) != cudaSuccess)
    return SPEC_ECUDA;
  WsHeader hdr = ws_header(scratch);
  GemmBuffers b{};
  b.arg_keys = reinterpret_cast<unsigned long long*>(static_cast<uint8_t*>(scratch) + kNoAllocHeader);
  b.ids = ids;
  b.maxv = maxlogit;
  b.tickets = hdr.tickets;
  b.status = hdr.status;
  // the same kernel choice as spec_lmhead_argmax (tcgen05 above 32 rows)
  return launch_gemm_any(p, kGemmArgmax, h, w, b, st) == cudaSuccess ? SPEC_OK : SPEC_ECUDA;
}

extern "C" int spec_noalloc_read_status(void* stream, unsigned* status) {
  if (!status) return SPEC_EINVAL;
  void* scratch = nullptr;
  int rc = scratch_for_current_device(&scratch);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned v = 0;
  if (cudaMemcpyAsync(&v, scratch, 4, cudaMemcpyDeviceToHost, st) != cudaSuccess) return SPEC_ECUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return SPEC_ECUDA;
  if (v && cudaMemsetAsync(scratch, 0, 4, st) != cudaSuccess) return SPEC_ECUDA;
  *status = v;
  if (v & SPEC_DEV_TIMEOUT) return SPEC_ETIMEOUT;
  return v ? SPEC_EDEVICE : SPEC_OK;
}

extern "C" int spec_noalloc_inject_status(unsigned bits, void* stream) {
  void* scratch = nullptr;
  int rc = scratch_for_current_device(&scratch);
  if (rc) return rc;
  return launch_k(noalloc_inject_kernel, dim3(1), dim3(1), 0, static_cast<cudaStream_t>(stream),
                  ws_header(scratch).status, bits) == cudaSuccess
             ? SPEC_OK
             : SPEC_ECUDA;
}

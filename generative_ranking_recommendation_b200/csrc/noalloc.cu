// genrank_attn_fwd_static: the attention forward for callers that cannot allocate
// device memory.
//
// Some callers cannot call cudaMalloc (or any allocator) at the point where they
// run attention: code that runs inside a host-side allocation-free region, such as
// a real-time serving loop with a hard rule against device allocations after
// start-up, or an embedding in a framework that owns all device memory and hands
// out no scratch.  For them this entry point takes its scratch from a fixed
// array compiled into the library instead of a caller workspace.  Everything
// else (inputs and outputs) is still passed by the caller.
//
// The scratch is a file-scope __device__ array of kStaticScratchBytes (16 MiB).
// Every GPU on which the library is loaded holds it until the process exits.
// Host code cannot use the array's name as a device address; its address is
// looked up once per device with cudaGetSymbolAddress, with that device current.
#include "common.cuh"
#include "host_util.h"
#include "kernels.h"

namespace gr {
namespace {

constexpr size_t kStaticScratchBytes = size_t(16) << 20;

static __device__ __align__(256) uint8_t g_attn_scratch[kStaticScratchBytes];

void* g_scratch_addr[kMaxDevices] = {};

// Address of the scratch array on the current device, looked up once per device (with
// that device current) by cudaGetSymbolAddress.
void* scratch_for_current_device(int* code) {
  static DeviceOnce once;
  const int ok = once.run([](int dev) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_attn_scratch) != cudaSuccess || !p) return 0;
    g_scratch_addr[dev] = p;
    return 1;
  });
  int dev = 0;
  if (ok != 1 || cudaGetDevice(&dev) != cudaSuccess) {
    *code = GENRANK_ERR_CUDA;
    return nullptr;
  }
  *code = GENRANK_OK;
  return g_scratch_addr[dev];
}

}  // namespace
}  // namespace gr

extern "C" {

int genrank_attn_fwd_static(int B, int64_t T, const int32_t* seq_offsets,
                            const int32_t* hist_len, int max_seqlen, const void* q, const void* k,
                            const void* v, int64_t tok_stride, int H, int dh, const int32_t* pos,
                            const int64_t* ts, const float* slope_pos, const float* slope_time,
                            float scale, int dtype, void* o, int64_t o_stride, float* lse,
                            int32_t* dev_err, genrank_stream_t stream) {
  if (B < 1 || T < 0 || H < 1 || dh < 1 || max_seqlen < 0) return GENRANK_ERR_INVALID_ARG;
  const size_t need = genrank_attn_workspace_size(B, T, H, dh, max_seqlen, 0);
  if (need == 0) return GENRANK_ERR_INVALID_ARG;
  // only the tensor-core kernel (bf16, head dim 64) uses scratch; the CUDA-core kernel
  // runs without any, whatever the sizes
  const bool uses_scratch = dtype == GENRANK_BF16 && dh == 64;
  if (uses_scratch && need > gr::kStaticScratchBytes) return GENRANK_ERR_WORKSPACE;
  int code = GENRANK_OK;
  void* ws = gr::scratch_for_current_device(&code);
  if (code != GENRANK_OK) return code;
  // Nothing in the scratch has to start at zero: the forward writes the work list and
  // its count before reading them, and column terms left from an earlier call are only
  // ever read for keys that the mask removes.
  return genrank_attn_fwd(B, T, seq_offsets, hist_len, max_seqlen, q, k, v, tok_stride, H, dh,
                          pos, ts, slope_pos, slope_time, scale, dtype, o, o_stride, lse, ws,
                          gr::kStaticScratchBytes, dev_err, stream);
}

}  // extern "C"

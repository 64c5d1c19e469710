// Allocation-free variant of fastnn_reciprocal.
//
// Who needs it: code that must not call cudaMalloc while it runs. Examples are
// a plugin living inside a host application that owns every device allocation
// (a serving runtime or game engine with its own pool), a real-time loop where
// cudaMalloc's implicit device synchronisation would break latency, and
// callers with a fixed, pre-reserved memory budget. Such callers cannot
// provide the workspace that fastnn_reciprocal asks for, so this entry point
// keeps its scratch in a file-scope device array instead.
//
// The array is a static __device__ symbol: it exists on every GPU that loads
// this library, from module load until process exit, whether or not this
// entry point is ever called. Host code only sees a stand-in for it, so its
// device address is fetched with cudaGetSymbolAddress, once per device, with
// that device current; that happens on the first call made on each device.
#include <mutex>

#include "common.cuh"

namespace {

constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[FASTNN_NOALLOC_SCRATCH_BYTES];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (first call per
// device looks it up). Returns nullptr on failure.
void* scratch_for_current_device() {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    fastnn::note_cuda_error(e);
    return nullptr;
  }
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) {
      fastnn::note_cuda_error(e);
      return nullptr;
    }
    g_noalloc_ptr[dev] = p;
  }
  return g_noalloc_ptr[dev];
}

}  // namespace

extern "C" int fastnn_reciprocal_noalloc(const void* desc1, int H1, int W1, const void* desc2,
                                         int H2, int W2, int d, int dtype, int subsample,
                                         int max_iter, int batch, int32_t* out_pairs,
                                         void* out_score, int64_t capacity, int32_t* out_count,
                                         int32_t* out_iters, int32_t* out_frontier,
                                         fastnn_stream_t stream) {
  // Every argument check runs before the scratch lookup (the first CUDA call),
  // in fastnn_reciprocal's order, so that both entry points return the same
  // status for the same bad arguments.
  const bool dtype_ok = dtype == FASTNN_I8 || dtype == FASTNN_BF16 || dtype == FASTNN_F16 ||
                        dtype == FASTNN_F32_L2;
  if (!dtype_ok || d < 1 || d > (dtype == FASTNN_F32_L2 ? 3 : 64)) return FASTNN_ERR_UNSUPPORTED;
  if (subsample < 1 || H1 < 1 || W1 < 1 || H2 < 1 || W2 < 1 || batch < 1 || max_iter < 1 ||
      max_iter > 255)
    return FASTNN_ERR_INVALID;
  if (!desc1 || !desc2 || !out_pairs || !out_count) return FASTNN_ERR_INVALID;
  const int64_t S = static_cast<int64_t>((H1 + subsample - 1) / subsample) *
                    ((W1 + subsample - 1) / subsample);
  if (capacity < S) return FASTNN_ERR_CAPACITY;
  const size_t need =
      fastnn_workspace_size(FASTNN_OP_RECIPROCAL, static_cast<int64_t>(H1) * W1,
                            static_cast<int64_t>(H2) * W2, d, dtype, batch, S);
  if (need == 0) return FASTNN_ERR_INVALID;
  if (need > FASTNN_NOALLOC_SCRATCH_BYTES) return FASTNN_ERR_CAPACITY;
  void* scratch = scratch_for_current_device();
  if (!scratch) return FASTNN_ERR_CUDA;
  // Everything the computation reads before writing is cleared by
  // fastnn_reciprocal itself on the stream, so the previous call's contents
  // left in the array do no harm.
  return fastnn_reciprocal(desc1, H1, W1, desc2, H2, W2, d, dtype, subsample, max_iter, batch,
                           out_pairs, out_score, capacity, out_count, out_iters, out_frontier,
                           scratch, need, stream);
}

// The status word sits at the head of the scratch array, where
// fastnn_reciprocal keeps it at the head of any workspace.
extern "C" int fastnn_noalloc_device_status(fastnn_stream_t stream) {
  void* scratch = scratch_for_current_device();
  if (!scratch) return FASTNN_ERR_CUDA;
  return fastnn_device_status(scratch, stream);
}

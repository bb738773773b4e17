// muse_cluster_static: the k-means entry point for callers that cannot
// allocate device memory.
//
// Some callers have no way to hand the library a workspace: code that runs
// where cudaMalloc is not allowed or not safe (for example a serving process
// whose device memory is fully planned at start-up and that must not grow
// it per request, or a host thread that has no allocator of its own), and C
// callers that only hold the input and output buffers.  This entry point
// takes the k-means scratch from a fixed array compiled into the library
// instead, so it allocates nothing itself.
//
// The array is a file-scope __device__ symbol of kStaticScratchBytes: every
// GPU that loads the library holds it until the process exits.  In host code
// the symbol's name is only a host-side stand-in, so its device address is
// looked up once per device with cudaGetSymbolAddress (on the first call made
// on that device, with that device current) and passed to the kernels; the
// address is kept for the life of the process, so it is stale after a
// cudaDeviceReset() of that device.
// Every call shares the array and it keeps the last call's contents; the
// parts that must start at zero (tile arrival counters, the error word) are
// cleared on the stream by each call.  Calls whose work overlaps on the GPU
// (different streams, or concurrent host threads) race on the array.
#include <cuda_runtime.h>

#include <mutex>
#include <string>

#include "../../include/muse.h"

namespace {

constexpr size_t kStaticScratchBytes = (size_t)16 << 20;  // 16 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_scratch[kStaticScratchBytes];

std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {nullptr};

}  // namespace

namespace muse {
void set_last_error(const char* msg);  // the message muse_last_error() returns
}

extern "C" {

size_t muse_cluster_static_capacity(void) { return kStaticScratchBytes; }

muse_status muse_cluster_static(const void* X, muse_dtype dtype, int B, int H, int N, int D,
                                int C, int iters, uint64_t seed, int role, const float* init,
                                int32_t* assign, float* centroids, int32_t* counts,
                                int32_t* device_error, cudaStream_t stream) {
  const size_t need = muse_cluster_workspace_size(B, H, N, D, C);
  if (need > kStaticScratchBytes) {
    // rejected before touching the device; argument errors are left to muse_cluster
    const std::string msg = "muse_cluster_static: these sizes need " + std::to_string(need) +
                            " bytes of scratch, more than the " +
                            std::to_string(kStaticScratchBytes) +
                            " bytes built into the library; use muse_cluster with a workspace";
    muse::set_last_error(msg.c_str());
    return MUSE_ERR_WORKSPACE;
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    muse::set_last_error("muse_cluster_static: no current CUDA device");
    return MUSE_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    muse::set_last_error("muse_cluster_static: device index beyond the supported 64");
    return MUSE_ERR_UNSUPPORTED;
  }
  void* ws = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_scratch_addr[dev] == nullptr) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || p == nullptr) {
        cudaGetLastError();
        muse::set_last_error("muse_cluster_static: cudaGetSymbolAddress of the scratch failed");
        return MUSE_ERR_CUDA;
      }
      g_scratch_addr[dev] = p;
    }
    ws = g_scratch_addr[dev];
  }
  return muse_cluster(X, dtype, B, H, N, D, C, iters, seed, role, init, assign, centroids, counts,
                      device_error, ws, kStaticScratchBytes, stream);
}

}  // extern "C"

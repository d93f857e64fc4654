// wal_gemm_tc_noalloc: the tensor-core product with its scratch in a fixed
// array of the library's own device memory instead of a caller workspace.
// The model cards have no counterpart; this exists for callers that cannot
// hand the library scratch memory.  Nothing here allocates: the array is a
// file-scope device variable, located with cudaGetSymbolAddress on every call
// (so the address always belongs to the current device and context).  Every
// call on a device shares it, so calls that overlap in time on one device race
// on it.  wal_noalloc_status reads the status word at its head.
#include "wal_internal.h"
#include "wal_stream.h"
#include "wal_tc.h"

namespace wal {

int check_product_args(const wal_matrix* m, const void* X, int M, int ldx, const void* Y, int ldy);

namespace {

constexpr size_t kScratchBytes = WAL_NOALLOC_SCRATCH_BYTES;  // 16 MiB

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

// Device address of the scratch array on the current device.
int scratch_base(char** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_scratch);
  if (e != cudaSuccess) return fail(WAL_ERR_CUDA, std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e));
  *out = static_cast<char*>(p);
  return WAL_OK;
}

}  // namespace
}  // namespace wal

using namespace wal;

extern "C" int wal_gemm_tc_noalloc(const wal_matrix* m, const uint16_t* X, int M, int ldx, float* Y, int ldy,
                                   wal_stream_t stream) {
  int st = check_product_args(m, X, M, ldx, Y, ldy);
  if (st) return st;
  if (M < kTcMinM) return fail(WAL_ERR_SHAPE, "wal_gemm_tc_noalloc takes M >= 5 (the tensor-core path)");
  const size_t need = tc_ws_bytes(m, M);
  if (need == 0 || need > kScratchBytes)
    return fail(WAL_ERR_WORKSPACE, "scratch need above the fixed 16 MiB array");
  char* base = nullptr;
  st = scratch_base(&base);
  if (st) return st;
  // the header's status word must start at zero; every other scratch byte is
  // written by the prep kernel before it is read
  cudaError_t e = cudaMemsetAsync(base, 0, 256, (cudaStream_t)stream);
  if (e != cudaSuccess) return fail(WAL_ERR_CUDA, std::string("scratch header clear: ") + cudaGetErrorString(e));
  return launch_tc(m, X, M, ldx, Y, ldy, base, (cudaStream_t)stream);
}

extern "C" int wal_noalloc_status(wal_stream_t stream) {
  char* base = nullptr;
  int st = scratch_base(&base);
  if (st) return st;
  int32_t h = 0;
  const cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaMemcpyAsync(&h, base, 4, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(base, 0, 4, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return fail(WAL_ERR_CUDA, std::string("scratch status readback: ") + cudaGetErrorString(e));
  if (h != 0) return fail(WAL_ERR_TIMEOUT, "a bounded device wait gave up");
  return WAL_OK;
}

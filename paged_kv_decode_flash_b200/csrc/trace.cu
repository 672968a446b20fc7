// trace.cu -- set-up and completion of the key-resolution record that the
// decode kernel writes when it is launched with a trace buffer (the record
// itself comes from the kernel that reads the cache: every (row, key) pair
// it scores, with the physical slot its K row was copied from).  Tests only.
#include <climits>

#include "common.cuh"
#include "kernels.h"

namespace pa {
namespace {

__global__ void trace_init_kernel(int32_t* trace, long long rows) {
  const long long r = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= rows) return;
  int32_t* t = trace + r * 5;
  t[0] = 0; t[1] = INT_MAX; t[2] = -1; t[3] = 0; t[4] = 0;
}

__global__ void trace_finish_kernel(int32_t* trace, long long rows) {
  const long long r = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= rows) return;
  int32_t* t = trace + r * 5;
  if (t[0] == 0) t[1] = -1;  // a row no key reached: {0, -1, -1, 0, 0}
}

}  // namespace

cudaError_t launch_trace_init(int32_t* trace, long long rows, cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  trace_init_kernel<<<(unsigned)((rows + 127) / 128), 128, 0, stream>>>(trace, rows);
  return cudaGetLastError();
}

cudaError_t launch_trace_finish(int32_t* trace, long long rows, cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  trace_finish_kernel<<<(unsigned)((rows + 127) / 128), 128, 0, stream>>>(trace, rows);
  return cudaGetLastError();
}

}  // namespace pa

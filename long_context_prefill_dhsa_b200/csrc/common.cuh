// Internal helpers shared by the DHSA kernels and the C-ABI layer.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "../../include/dhsa.h"

namespace dhsa {

constexpr int kHeadDim = 128;
constexpr int kQueryTileRows = 128;   // query rows per attention tile

// Device address of the current device's status word (bits DHSA_DEVFLAG_*),
// or nullptr with the CUDA error recorded. Kernels that can fail on the device
// take this pointer as an argument and atomically OR their flag into it.
unsigned int* device_status_ptr();

__device__ __forceinline__ void raise_device_flag(unsigned int* status, unsigned int bit) {
  atomicOr(status, bit);
}

// Host side: remember the CUDA error behind a DHSA_ERR_CUDA.
void set_last_cuda_error(cudaError_t e);

inline int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return DHSA_OK;
  set_last_cuda_error(e);
  return DHSA_ERR_CUDA;
}

// Wall-clock limit of every bounded device wait (1 s).
constexpr unsigned long long kWaitLimitNs = 1000000000ull;

// Test hook of the bounded waits: true (once) when dhsa_debug_arm_wait_timeout
// armed `mode` (1 = attention, 2 = fused routing); *limit_ns gets the short
// limit the launch must use. Host side, not thread-safe.
bool take_wait_test(int mode, unsigned long long* limit_ns);

// Launch check: picks up configuration errors of the launch just made.
inline int launch_status() { return cuda_status(cudaGetLastError()); }

// The library is built for sm_100a only.
int check_device_sm100();

__host__ __device__ inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Block CSR written by the top-k selection itself (row_ptr null: none).
struct CsrOut {
  int32_t* row_ptr;
  int32_t* col_idx;
  int64_t* cost;        // may be null
  const int32_t* off;
  unsigned int* status;
};

}  // namespace dhsa

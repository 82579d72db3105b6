// Attention forward over the kept chunk pairs: builds the work lists of the
// tile policy (0: 128-row tiles only; 1: chunk tails of at most 64 rows on
// the short-tile kernel; 2: 64-row tiles only) and launches the long-tile
// kernel (attn_fwd.cu, 128 query rows per tile) and the short-tile kernel
// (attn_short.cu, at most 64 rows) on one stream. The two write disjoint
// rows of O.
#include "common.cuh"
#include "tmap.cuh"

namespace dhsa {

long long attn_cap_long(int B, int Hq, int L, int Nmax, int policy);
long long attn_cap_short(int B, int Hq, int L, int Nmax, int policy);
int launch_build_items(const int32_t* off, const int32_t* n_chunks, int B, int Hq, int G, int L, int Nmax,
                       int policy, const AttnWork& w, unsigned int* status, cudaStream_t stream);
int launch_sparse_attn_long(const AttnWork& w, const void* Q, const void* K, const void* V, int B, int Hq, int Hkv,
                            int L, const int32_t* off, int Nmax, const int32_t* row_ptr, const int32_t* col_idx,
                            float softmax_scale, void* O, unsigned int* status, cudaStream_t stream);
int launch_sparse_attn_short(const AttnWork& w, const void* Q, const void* K, const void* V, int B, int Hq, int Hkv,
                             int L, const int32_t* off, int Nmax, const int32_t* row_ptr, const int32_t* col_idx,
                             float softmax_scale, void* O, unsigned int* status, cudaStream_t stream);

// workspace: [0] long count, [1] long dispenser, [2] short count, [3] short
// dispenser; the long list from byte 256, the short list after it
size_t attn_ws_bytes(int B, int Hq, int L, int Nmax, int policy) {
  return 256 + sizeof(int4) * (size_t)(attn_cap_long(B, Hq, L, Nmax, policy) + attn_cap_short(B, Hq, L, Nmax, policy));
}

int launch_sparse_attn(const void* Q, const void* K, const void* V, int B, int Hq, int Hkv, int L,
                       const int32_t* off, const int32_t* n_chunks, int Nmax, const int32_t* row_ptr,
                       const int32_t* col_idx, float softmax_scale, int policy, void* O, void* ws,
                       unsigned int* status, cudaStream_t stream) {
  int* head = static_cast<int*>(ws);
  AttnWork w;
  w.cap_long = attn_cap_long(B, Hq, L, Nmax, policy);
  w.cap_short = attn_cap_short(B, Hq, L, Nmax, policy);
  w.n_long = head;
  w.counter_long = head + 1;
  w.n_short = head + 2;
  w.counter_short = head + 3;
  w.items_long = reinterpret_cast<int4*>(static_cast<char*>(ws) + 256);
  w.items_short = w.items_long + w.cap_long;
  int st = launch_build_items(off, n_chunks, B, Hq, Hq / Hkv, L, Nmax, policy, w, status, stream);
  if (st == DHSA_OK)
    st = launch_sparse_attn_long(w, Q, K, V, B, Hq, Hkv, L, off, Nmax, row_ptr, col_idx, softmax_scale, O, status,
                                 stream);
  if (st == DHSA_OK)
    st = launch_sparse_attn_short(w, Q, K, V, B, Hq, Hkv, L, off, Nmax, row_ptr, col_idx, softmax_scale, O,
                                  status, stream);
  return st;
}

// ----------------------------------------------------------- no-allocation variant
// Scratch for callers that must not allocate device memory. It lives in a
// file-scope device array that every GPU loading the library holds until the
// process exits. It backs the same work lists the caller's workspace would
// hold, so the largest problem is the one whose attn_ws_bytes is <= 4 MiB.
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
constexpr int kNoAllocMaxDevices = 64;
void* g_noalloc_ptr[kNoAllocMaxDevices] = {nullptr};
}  // namespace

size_t noalloc_scratch_bytes() { return kNoAllocScratchBytes; }

// Device address of the static scratch on the current device. The host-side
// name g_noalloc_scratch is only a stand-in, so the address is looked up once
// per device (on that device's first call) and cached.
int noalloc_scratch_ptr(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_status(e);
  if (dev < 0 || dev >= kNoAllocMaxDevices) return DHSA_ERR_UNSUPPORTED;
  if (!g_noalloc_ptr[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_status(e);
    g_noalloc_ptr[dev] = ptr;
  }
  *out = g_noalloc_ptr[dev];
  return DHSA_OK;
}

}  // namespace dhsa

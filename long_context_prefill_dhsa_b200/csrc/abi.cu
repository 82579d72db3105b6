// extern "C" entry points of libdhsa: host-side argument checks, then the
// stage launchers. Every check happens before anything is enqueued.
#include <cstring>

#include "common.cuh"

namespace dhsa {

int launch_chunk_pool(const void* X, int B, int H, int L, const int32_t* off, const int32_t* n_chunks, int Nmax,
                      float* Xp, unsigned int* status, cudaStream_t stream);
int launch_chunk_pool_qk(const void* Q, const void* K, int B, int Hq, int Hkv, int L, const int32_t* off,
                         const int32_t* n_chunks, int Nmax, float* Qp, float* Kp, unsigned int* status,
                         cudaStream_t stream);
int launch_validate_offsets(const int32_t* off, const int32_t* n_chunks, int B, int Nmax, int L,
                            unsigned int* status, cudaStream_t stream);
int score_topk_stride(int k, int Nmax);
size_t score_topk_ws_bytes(int B, int Hq, int Nmax);
int launch_score_topk(const float* Qp, const float* Kp, int B, int Hq, int Hkv, int Nmax, const int32_t* n_chunks,
                      int k, int32_t* sel, int32_t* n_sel, void* ws, const CsrOut& csr, cudaStream_t stream);
int launch_route_fused(const void* Q, const void* K, int B, int Hq, int Hkv, int L, const int32_t* off,
                       const int32_t* n_chunks, int Nmax, int k, float* Qp, float* Kp, int32_t* sel, int32_t* n_sel,
                       const CsrOut& csr, void* ws, unsigned int* status, unsigned long long limit_ns,
                       unsigned long long hold_ns, cudaStream_t stream);
int score_budget_max_chunks();
int launch_score_budget(const float* Qp, const float* Kp, int B, int Hq, int Hkv, int Nmax, const int32_t* off,
                        const int32_t* n_chunks, int budget, const int32_t* budgets, int recent, int k_max,
                        int32_t* sel, int32_t* n_sel, void* ws, cudaStream_t stream);
int launch_build_csr(const int32_t* sel, const int32_t* n_sel, int B, int Hq, int Nmax, int k, const int32_t* off,
                     const int32_t* n_chunks, int32_t* row_ptr, int32_t* col_idx, int64_t* cost,
                     unsigned int* status, cudaStream_t stream);
size_t attn_ws_bytes(int B, int Hq, int L, int Nmax, int policy);
int launch_sparse_attn(const void* Q, const void* K, const void* V, int B, int Hq, int Hkv, int L,
                       const int32_t* off, const int32_t* n_chunks, int Nmax, const int32_t* row_ptr,
                       const int32_t* col_idx, float softmax_scale, int policy, void* O, void* ws,
                       unsigned int* status, cudaStream_t stream);
size_t noalloc_scratch_bytes();
int noalloc_scratch_ptr(void** out);

namespace {
__device__ unsigned int g_device_status = 0;
thread_local int t_last_cuda_error = 0;
constexpr int kMaxDevices = 64;
unsigned int* g_status_ptr[kMaxDevices] = {nullptr};
int g_sm100[kMaxDevices] = {0};  // 0 unknown, 1 yes, -1 no

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
}  // namespace

void set_last_cuda_error(cudaError_t e) { t_last_cuda_error = (int)e; }

namespace {
// armed test hook of the bounded waits (dhsa_debug_arm_wait_timeout)
int g_wait_test_mode = 0;
unsigned long long g_wait_test_limit_ns = 0;
}  // namespace

bool take_wait_test(int mode, unsigned long long* limit_ns) {
  if (g_wait_test_mode != mode) return false;
  *limit_ns = g_wait_test_limit_ns;
  g_wait_test_mode = 0;
  return true;
}

unsigned int* device_status_ptr() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    set_last_cuda_error(e == cudaSuccess ? cudaErrorInvalidDevice : e);
    return nullptr;
  }
  if (!g_status_ptr[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_device_status);
    if (e != cudaSuccess) {
      set_last_cuda_error(e);
      return nullptr;
    }
    g_status_ptr[dev] = static_cast<unsigned int*>(ptr);
  }
  return g_status_ptr[dev];
}

int check_device_sm100() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_status(e);
  if (dev < 0 || dev >= kMaxDevices) return DHSA_ERR_UNSUPPORTED;
  if (g_sm100[dev] == 0) {
    int major = 0, minor = 0;
    e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (e != cudaSuccess) return cuda_status(e);
    g_sm100[dev] = (major == 10 && minor == 0) ? 1 : -1;
  }
  return g_sm100[dev] == 1 ? DHSA_OK : DHSA_ERR_UNSUPPORTED;
}

}  // namespace dhsa

using namespace dhsa;

namespace {
int check_layout(int B, int H, int L, int Nmax, const int32_t* off, const int32_t* n_chunks) {
  if (B <= 0 || H <= 0 || L <= 0 || Nmax <= 0 || Nmax > L) return DHSA_ERR_INVALID_ARG;
  if (!off || !n_chunks) return DHSA_ERR_INVALID_ARG;
  if ((long long)B * H * L > 0x7fffffffLL) return DHSA_ERR_INVALID_ARG;  // TMA row coordinates are int32
  return DHSA_OK;
}
}  // namespace

extern "C" {

const char* dhsa_status_string(int status) {
  switch (status) {
    case DHSA_OK: return "DHSA_OK";
    case DHSA_ERR_INVALID_ARG: return "DHSA_ERR_INVALID_ARG";
    case DHSA_ERR_UNSUPPORTED: return "DHSA_ERR_UNSUPPORTED";
    case DHSA_ERR_CUDA: return "DHSA_ERR_CUDA";
    case DHSA_ERR_DEVICE: return "DHSA_ERR_DEVICE";
    case DHSA_ERR_WORKSPACE: return "DHSA_ERR_WORKSPACE";
    default: return "DHSA_ERR_UNKNOWN";
  }
}

int dhsa_last_cuda_error(void) { return t_last_cuda_error; }

int dhsa_version(void) { return 300; }   // 0.3.0: wait-timeout test hook; offsets clamped by pooling and the work list

int dhsa_check_device_status(void* stream, uint32_t* device_flags) {
  if (device_flags) *device_flags = 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_status(e);
  unsigned int* ptr = device_status_ptr();
  if (!ptr) return DHSA_ERR_CUDA;
  unsigned int flags = 0;
  e = cudaMemcpyAsync(&flags, ptr, sizeof(flags), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(ptr, 0, sizeof(unsigned int), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_status(e);
  if (device_flags) *device_flags = flags;
  return flags ? DHSA_ERR_DEVICE : DHSA_OK;
}

int dhsa_validate_offsets(const int32_t* off, const int32_t* n_chunks, int B, int Nmax, int L, void* stream) {
  int st = check_layout(B, 1, L, Nmax, off, n_chunks);
  if (st != DHSA_OK) return st;
  if ((st = check_device_sm100()) != DHSA_OK) return st;
  unsigned int* status = device_status_ptr();
  if (!status) return DHSA_ERR_CUDA;
  return launch_validate_offsets(off, n_chunks, B, Nmax, L, status, static_cast<cudaStream_t>(stream));
}

int dhsa_chunk_pool(const void* X, int B, int H, int L, int head_dim, const int32_t* off, const int32_t* n_chunks,
                    int Nmax, float* Xp, void* stream) {
  int st = check_layout(B, H, L, Nmax, off, n_chunks);
  if (st != DHSA_OK) return st;
  if (!X || !Xp || !aligned16(X) || !aligned16(Xp)) return DHSA_ERR_INVALID_ARG;
  if (head_dim != kHeadDim) return DHSA_ERR_UNSUPPORTED;
  if ((st = check_device_sm100()) != DHSA_OK) return st;
  unsigned int* status = device_status_ptr();
  if (!status) return DHSA_ERR_CUDA;
  return launch_chunk_pool(X, B, H, L, off, n_chunks, Nmax, Xp, status, static_cast<cudaStream_t>(stream));
}

int dhsa_chunk_pool_qk(const void* Q, const void* K, int B, int Hq, int Hkv, int L, int head_dim,
                       const int32_t* off, const int32_t* n_chunks, int Nmax, float* Qp, float* Kp, void* stream) {
  int st = check_layout(B, Hq, L, Nmax, off, n_chunks);
  if (st != DHSA_OK) return st;
  if (Hkv <= 0 || Hq % Hkv != 0) return DHSA_ERR_INVALID_ARG;
  if (!Q || !K || !Qp || !Kp || !aligned16(Q) || !aligned16(K) || !aligned16(Qp) || !aligned16(Kp))
    return DHSA_ERR_INVALID_ARG;
  if (head_dim != kHeadDim) return DHSA_ERR_UNSUPPORTED;
  if ((st = check_device_sm100()) != DHSA_OK) return st;
  unsigned int* status = device_status_ptr();
  if (!status) return DHSA_ERR_CUDA;
  return launch_chunk_pool_qk(Q, K, B, Hq, Hkv, L, off, n_chunks, Nmax, Qp, Kp, status,
                              static_cast<cudaStream_t>(stream));
}

int dhsa_sel_stride(int k, int Nmax) {
  if (k < 0 || Nmax <= 0) return 0;
  return score_topk_stride(k, Nmax);
}

size_t dhsa_score_topk_workspace_size(int B, int Hq, int Nmax) {
  if (B <= 0 || Hq <= 0 || Nmax <= 0) return 0;
  return score_topk_ws_bytes(B, Hq, Nmax);
}

int dhsa_chunk_score_topk(const float* Qp, const float* Kp, int B, int Hq, int Hkv, int Nmax,
                          const int32_t* n_chunks, int k, int32_t* sel, int32_t* n_sel, void* workspace,
                          size_t workspace_bytes, void* stream) {
  if (!Qp || !Kp || !n_chunks || !sel || !n_sel) return DHSA_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nmax <= 0 || k < 0 || Hq % Hkv != 0) return DHSA_ERR_INVALID_ARG;
  const size_t need = score_topk_ws_bytes(B, Hq, Nmax);
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return DHSA_ERR_WORKSPACE;
  int st = check_device_sm100();
  if (st != DHSA_OK) return st;
  const CsrOut none{nullptr, nullptr, nullptr, nullptr, nullptr};
  return launch_score_topk(Qp, Kp, B, Hq, Hkv, Nmax, n_chunks, k, sel, n_sel, workspace, none,
                           static_cast<cudaStream_t>(stream));
}

int dhsa_chunk_score_topk_csr(const float* Qp, const float* Kp, int B, int Hq, int Hkv, int Nmax,
                              const int32_t* off, const int32_t* n_chunks, int k, int32_t* sel, int32_t* n_sel,
                              int32_t* row_ptr, int32_t* col_idx, int64_t* cost, void* workspace,
                              size_t workspace_bytes, void* stream) {
  if (!Qp || !Kp || !off || !n_chunks || !sel || !n_sel || !row_ptr || !col_idx) return DHSA_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nmax <= 0 || k < 0 || Hq % Hkv != 0) return DHSA_ERR_INVALID_ARG;
  if (dhsa_csr_nnz_upper(B, Hq, Nmax, k) > 0x7fffffffULL) return DHSA_ERR_INVALID_ARG;   // int32 row_ptr
  const size_t need = score_topk_ws_bytes(B, Hq, Nmax);
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return DHSA_ERR_WORKSPACE;
  int st = check_device_sm100();
  if (st != DHSA_OK) return st;
  unsigned int* status = device_status_ptr();
  if (!status) return DHSA_ERR_CUDA;
  const CsrOut csr{row_ptr, col_idx, cost, off, status};
  return launch_score_topk(Qp, Kp, B, Hq, Hkv, Nmax, n_chunks, k, sel, n_sel, workspace, csr,
                           static_cast<cudaStream_t>(stream));
}

size_t dhsa_route_fused_workspace_size(int B, int Hq, int Nmax) {
  if (B <= 0 || Hq <= 0 || Nmax <= 0) return 0;
  return score_topk_ws_bytes(B, Hq, Nmax);
}

namespace {
int route_fused_common(const void* Q, const void* K, int B, int Hq, int Hkv, int L, int head_dim, const int32_t* off,
                       const int32_t* n_chunks, int Nmax, int k, float* Qp, float* Kp, int32_t* sel, int32_t* n_sel,
                       int32_t* row_ptr, int32_t* col_idx, int64_t* cost, void* workspace, size_t workspace_bytes,
                       void* stream) {
  int st = check_layout(B, Hq, L, Nmax, off, n_chunks);
  if (st != DHSA_OK) return st;
  if (Hkv <= 0 || Hq % Hkv != 0 || k < 0) return DHSA_ERR_INVALID_ARG;
  if (!Q || !K || !Qp || !Kp || !sel || !n_sel || !aligned16(Q) || !aligned16(K) || !aligned16(Qp) ||
      !aligned16(Kp))
    return DHSA_ERR_INVALID_ARG;
  if (head_dim != kHeadDim) return DHSA_ERR_UNSUPPORTED;
  const size_t need = score_topk_ws_bytes(B, Hq, Nmax);
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return DHSA_ERR_WORKSPACE;
  if ((st = check_device_sm100()) != DHSA_OK) return st;
  unsigned int* status = device_status_ptr();
  if (!status) return DHSA_ERR_CUDA;
  unsigned long long limit_ns = kWaitLimitNs, hold_ns = 0, test_ns = 0;
  if (take_wait_test(2, &test_ns)) {   // block 0 arrives late; the others give up after test_ns
    limit_ns = test_ns;
    hold_ns = 4 * test_ns + 1000000ull;
  }
  const CsrOut csr{row_ptr, col_idx, cost, off, status};
  return launch_route_fused(Q, K, B, Hq, Hkv, L, off, n_chunks, Nmax, k, Qp, Kp, sel, n_sel, csr, workspace, status,
                            limit_ns, hold_ns, static_cast<cudaStream_t>(stream));
}
}  // namespace

int dhsa_route_fused(const void* Q, const void* K, int B, int Hq, int Hkv, int L, int head_dim, const int32_t* off,
                     const int32_t* n_chunks, int Nmax, int k, float* Qp, float* Kp, int32_t* sel, int32_t* n_sel,
                     void* workspace, size_t workspace_bytes, void* stream) {
  return route_fused_common(Q, K, B, Hq, Hkv, L, head_dim, off, n_chunks, Nmax, k, Qp, Kp, sel, n_sel, nullptr,
                            nullptr, nullptr, workspace, workspace_bytes, stream);
}

int dhsa_route_topk_csr(const void* Q, const void* K, int B, int Hq, int Hkv, int L, int head_dim,
                        const int32_t* off, const int32_t* n_chunks, int Nmax, int k, float* Qp, float* Kp,
                        int32_t* sel, int32_t* n_sel, int32_t* row_ptr, int32_t* col_idx, int64_t* cost,
                        void* workspace, size_t workspace_bytes, void* stream) {
  if (!row_ptr || !col_idx) return DHSA_ERR_INVALID_ARG;
  if (B > 0 && Hq > 0 && Nmax > 0 && k >= 0 && dhsa_csr_nnz_upper(B, Hq, Nmax, k) > 0x7fffffffULL)
    return DHSA_ERR_INVALID_ARG;   // int32 row_ptr
  return route_fused_common(Q, K, B, Hq, Hkv, L, head_dim, off, n_chunks, Nmax, k, Qp, Kp, sel, n_sel, row_ptr,
                            col_idx, cost, workspace, workspace_bytes, stream);
}

int dhsa_budget_max_chunks(void) { return score_budget_max_chunks(); }

int dhsa_chunk_score_select_budget(const float* Qp, const float* Kp, int B, int Hq, int Hkv, int Nmax,
                                   const int32_t* off, const int32_t* n_chunks, int budget,
                                   const int32_t* budgets, int recent, int k_max, int32_t* sel, int32_t* n_sel,
                                   void* workspace, size_t workspace_bytes, void* stream) {
  if (!Qp || !Kp || !off || !n_chunks || !sel || !n_sel) return DHSA_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nmax <= 0 || Hq % Hkv != 0) return DHSA_ERR_INVALID_ARG;
  if (k_max < 0 || recent < 0 || (!budgets && budget < 0)) return DHSA_ERR_INVALID_ARG;
  if (k_max > score_budget_max_chunks()) return DHSA_ERR_UNSUPPORTED;
  const size_t need = score_topk_ws_bytes(B, Hq, Nmax);
  if (need && (!workspace || workspace_bytes < need || !aligned16(workspace))) return DHSA_ERR_WORKSPACE;
  int st = check_device_sm100();
  if (st != DHSA_OK) return st;
  return launch_score_budget(Qp, Kp, B, Hq, Hkv, Nmax, off, n_chunks, budget, budgets, recent, k_max, sel, n_sel,
                             need ? workspace : nullptr, static_cast<cudaStream_t>(stream));
}

size_t dhsa_csr_nnz_upper(int B, int Hq, int Nmax, int k) {
  if (B <= 0 || Hq <= 0 || Nmax <= 0 || k < 0) return 0;
  return (size_t)B * Hq * Nmax * (size_t)score_topk_stride(k, Nmax);
}

int dhsa_build_block_csr(const int32_t* sel, const int32_t* n_sel, int B, int Hq, int Nmax, int k,
                         const int32_t* off, const int32_t* n_chunks, int32_t* row_ptr, int32_t* col_idx,
                         int64_t* cost, void* stream) {
  if (!sel || !n_sel || !off || !n_chunks || !row_ptr || !col_idx) return DHSA_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Nmax <= 0 || k < 0) return DHSA_ERR_INVALID_ARG;
  if (dhsa_csr_nnz_upper(B, Hq, Nmax, k) > 0x7fffffffULL) return DHSA_ERR_INVALID_ARG;  // int32 row_ptr
  int st = check_device_sm100();
  if (st != DHSA_OK) return st;
  unsigned int* status = device_status_ptr();
  if (!status) return DHSA_ERR_CUDA;
  return launch_build_csr(sel, n_sel, B, Hq, Nmax, k, off, n_chunks, row_ptr, col_idx, cost, status,
                          static_cast<cudaStream_t>(stream));
}

size_t dhsa_sparse_attn_workspace_size(int B, int Hq, int L, int Nmax) {
  return dhsa_sparse_attn_tiles_workspace_size(B, Hq, L, Nmax, 0);
}

size_t dhsa_sparse_attn_tiles_workspace_size(int B, int Hq, int L, int Nmax, int short_tiles) {
  if (B <= 0 || Hq <= 0 || L <= 0 || Nmax <= 0 || short_tiles < 0 || short_tiles > 2) return 0;
  return attn_ws_bytes(B, Hq, L, Nmax, short_tiles);
}

int dhsa_sparse_attn_fwd(const void* Q, const void* K, const void* V, int B, int Hq, int Hkv, int L, int head_dim,
                         const int32_t* off, const int32_t* n_chunks, int Nmax, const int32_t* row_ptr,
                         const int32_t* col_idx, const int64_t* cost, float softmax_scale, void* O, void* workspace,
                         size_t workspace_bytes, void* stream) {
  (void)cost;
  return dhsa_sparse_attn_fwd_tiles(Q, K, V, B, Hq, Hkv, L, head_dim, off, n_chunks, Nmax, row_ptr, col_idx,
                                    softmax_scale, 0, O, workspace, workspace_bytes, stream);
}

int dhsa_sparse_attn_fwd_tiles(const void* Q, const void* K, const void* V, int B, int Hq, int Hkv, int L,
                               int head_dim, const int32_t* off, const int32_t* n_chunks, int Nmax,
                               const int32_t* row_ptr, const int32_t* col_idx, float softmax_scale, int short_tiles,
                               void* O, void* workspace, size_t workspace_bytes, void* stream) {
  int st = check_layout(B, Hq, L, Nmax, off, n_chunks);
  if (st != DHSA_OK) return st;
  if (!Q || !K || !V || !O || !row_ptr || !col_idx) return DHSA_ERR_INVALID_ARG;
  if (Hkv <= 0 || Hq % Hkv != 0) return DHSA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return DHSA_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.f) || softmax_scale != softmax_scale) return DHSA_ERR_INVALID_ARG;
  if (short_tiles < 0 || short_tiles > 2) return DHSA_ERR_INVALID_ARG;
  if (head_dim != kHeadDim) return DHSA_ERR_UNSUPPORTED;
  if (!workspace || workspace_bytes < attn_ws_bytes(B, Hq, L, Nmax, short_tiles) || !aligned16(workspace))
    return DHSA_ERR_WORKSPACE;
  if ((st = check_device_sm100()) != DHSA_OK) return st;
  unsigned int* status = device_status_ptr();
  if (!status) return DHSA_ERR_CUDA;
  return launch_sparse_attn(Q, K, V, B, Hq, Hkv, L, off, n_chunks, Nmax, row_ptr, col_idx, softmax_scale,
                            short_tiles, O, workspace, status, static_cast<cudaStream_t>(stream));
}

int dhsa_sparse_attn_fwd_noalloc(const void* Q, const void* K, const void* V, int B, int Hq, int Hkv, int L,
                                 int head_dim, const int32_t* off, const int32_t* n_chunks, int Nmax,
                                 const int32_t* row_ptr, const int32_t* col_idx, float softmax_scale, void* O,
                                 void* stream) {
  int st = check_layout(B, Hq, L, Nmax, off, n_chunks);
  if (st != DHSA_OK) return st;
  if (!Q || !K || !V || !O || !row_ptr || !col_idx) return DHSA_ERR_INVALID_ARG;
  if (Hkv <= 0 || Hq % Hkv != 0) return DHSA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return DHSA_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.f) || softmax_scale != softmax_scale) return DHSA_ERR_INVALID_ARG;
  if (head_dim != kHeadDim) return DHSA_ERR_UNSUPPORTED;
  if (attn_ws_bytes(B, Hq, L, Nmax, 0) > noalloc_scratch_bytes()) return DHSA_ERR_WORKSPACE;
  if ((st = check_device_sm100()) != DHSA_OK) return st;
  unsigned int* status = device_status_ptr();
  if (!status) return DHSA_ERR_CUDA;
  void* scratch = nullptr;
  if ((st = noalloc_scratch_ptr(&scratch)) != DHSA_OK) return st;
  return launch_sparse_attn(Q, K, V, B, Hq, Hkv, L, off, n_chunks, Nmax, row_ptr, col_idx, softmax_scale, 0, O,
                            scratch, status, static_cast<cudaStream_t>(stream));
}

int dhsa_debug_arm_wait_timeout(int mode, uint64_t limit_ns) {
  if (mode < 0 || mode > 2) return DHSA_ERR_INVALID_ARG;
  if (mode != 0 && (limit_ns == 0 || limit_ns > 100000000ull)) return DHSA_ERR_INVALID_ARG;
  g_wait_test_mode = mode;
  g_wait_test_limit_ns = limit_ns;
  return DHSA_OK;
}

}  // extern "C"

// Chunk similarity + causal per-query-chunk top-k (stages 2-3 of the DHSA routing).
//
// gist.science technical summary of "Long-Context Modeling with Dynamic
// Hierarchical Sparse Attention", "Hierarchical Routing Formulation": a
// chunk-level similarity matrix scores chunk-to-chunk interactions (Step 1)
// and each query chunk is routed to a compact set of key chunks under the
// causal constraint (Step 2). Here: S[i][j] = <Qp_i, Kp_j> for j < i, and the
// kept set is {i} + the min(k, i) earlier chunks ranked by (S desc, j asc).
//
// Layout of the work: one CTA of 8 warps owns 8 consecutive query chunks
// (rows) of one (b, hq). Scores are exact dot products of the fp32 pooled
// vectors accumulated in fp64 (fp32 x fp32 products are exact in fp64), so
// the ranking is decided on values within ~1e-7 relative of the real-number
// scores. Key tiles of 32 pooled rows are staged in shared memory as fp64;
// lane l of warp w scores key j0+l against row w. A row's scores stay in
// shared memory (or, for very many chunks, in a per-CTA workspace slice), and
// each warp then selects its row's top-k with an 8-pass, 8-bit radix select
// over an order-preserving 64-bit key, breaking ties at the threshold value
// by the lowest chunk index. The selected indices come out ascending.
#include "common.cuh"

namespace dhsa {
namespace {

constexpr int kRows = 8;          // query chunks per CTA (one per warp)
constexpr int kJT = 32;           // key chunks per staged tile
constexpr int kKsStride = kHeadDim + 1;
constexpr int kSmemScoreCap = 2048;  // largest Nmax whose row-block scores stay in shared memory
constexpr int kWsCtas = 512;      // CTAs of the workspace-backed path

__device__ __forceinline__ unsigned long long order_key(double s) {
  const unsigned long long u = (unsigned long long)__double_as_longlong(s);
  return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Top-m of keys(buf[0..n)) under (key desc, index asc), written ascending to out.
// Requires 0 < m < n. Returns the number written (= m); never writes past
// out[m-1]. hist: 256 ints of this warp's shared memory.
__device__ int warp_select_topm(const double* buf, int n, int m, int* hist, int32_t* out) {
  const int lane = threadIdx.x & 31;
  const unsigned full = 0xffffffffu;
  unsigned long long prefix = 0, mask = 0;
  int need = m;
  for (int shift = 56; shift >= 0; shift -= 8) {
    for (int q = lane; q < 256; q += 32) hist[q] = 0;
    __syncwarp();
    for (int j = lane; j < n; j += 32) {
      const unsigned long long kk = order_key(buf[j]);
      if ((kk & mask) == prefix) atomicAdd(&hist[(kk >> shift) & 255], 1);
    }
    __syncwarp();
    int c[8], lsum = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      c[q] = hist[255 - 8 * lane - q];
      lsum += c[q];
    }
    int incl = lsum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(full, incl, o);
      if (lane >= o) incl += t;
    }
    const int excl = incl - lsum;
    const unsigned ball = __ballot_sync(full, excl < need && need <= incl);
    const int src = __ffs(ball) - 1;
    int digit = 0, above = 0;
    if (lane == src) {
      int run = excl;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (run + c[q] >= need) {
          digit = 255 - 8 * lane - q;
          above = run;
          break;
        }
        run += c[q];
      }
    }
    digit = __shfl_sync(full, digit, src);
    above = __shfl_sync(full, above, src);
    prefix |= (unsigned long long)digit << shift;
    mask |= 0xFFull << shift;
    need -= above;
    __syncwarp();
  }
  // prefix is now the m-th largest key; take every larger key and the `need`
  // lowest-index keys equal to it, in ascending index order.
  int written = 0, eq_seen = 0;
  for (int j0 = 0; j0 < n; j0 += 32) {
    const int j = j0 + lane;
    const bool valid = j < n;
    const unsigned long long kk = valid ? order_key(buf[j]) : 0ull;
    const bool gt = valid && kk > prefix;
    const bool eq = valid && kk == prefix;
    const unsigned beq = __ballot_sync(full, eq);
    const bool take = gt || (eq && (eq_seen + __popc(beq & lanemask_lt())) < need);
    eq_seen += __popc(beq);
    const unsigned bt = __ballot_sync(full, take);
    const int pos = written + __popc(bt & lanemask_lt());
    if (take && pos < m) out[pos] = j;
    written += __popc(bt);
  }
  return written < m ? written : m;
}

__global__ void __launch_bounds__(256) score_topk_kernel(const float* __restrict__ Qp, const float* __restrict__ Kp,
                                                         int Hq, int G, int Nmax,
                                                         const int32_t* __restrict__ n_chunks, int k, int stride,
                                                         int32_t* __restrict__ sel, int32_t* __restrict__ n_sel,
                                                         long long n_blocks, double* __restrict__ ws) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  double* Qs = reinterpret_cast<double*>(smem_raw);                 // [kRows][128]
  double* Ks = Qs + kRows * kHeadDim;                               // [kJT][129]
  int* hist = reinterpret_cast<int*>(Ks + kJT * kKsStride);         // [kRows][256]
  double* sbuf = ws ? ws + (long long)blockIdx.x * kRows * Nmax
                    : reinterpret_cast<double*>(hist + kRows * 256);  // [kRows][Nmax]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int blocks_per_head = (Nmax + kRows - 1) / kRows;

  for (long long blk = blockIdx.x; blk < n_blocks; blk += gridDim.x) {
    const long long bh = blk / blocks_per_head;             // b * Hq + hq
    const int i0 = (int)(blk % blocks_per_head) * kRows;
    const int b = (int)(bh / Hq), hq = (int)(bh % Hq);
    const int n = n_chunks[b];
    const long long kv_row0 = ((long long)b * (Hq / G) + hq / G) * Nmax;

    // stage the block's pooled queries as fp64
    for (int idx = threadIdx.x; idx < kRows * kHeadDim; idx += blockDim.x) {
      const int r = idx / kHeadDim, d = idx % kHeadDim;
      const int i = i0 + r;
      Qs[idx] = (i < n) ? (double)Qp[(bh * Nmax + i) * kHeadDim + d] : 0.0;
    }
    const int i_last = min(i0 + kRows, n) - 1;               // largest real row in the block
    const int i = i0 + warp;
    double* row_scores = sbuf + warp * Nmax;
    for (int j0 = 0; j0 < i_last; j0 += kJT) {
      __syncthreads();
      for (int idx = threadIdx.x; idx < kJT * kHeadDim; idx += blockDim.x) {
        const int r = idx / kHeadDim, d = idx % kHeadDim;
        const int j = j0 + r;
        Ks[r * kKsStride + d] = (j < n) ? (double)Kp[(kv_row0 + j) * kHeadDim + d] : 0.0;
      }
      __syncthreads();
      const int j = j0 + lane;
      if (i < n && j < i) {
        const double* q = Qs + warp * kHeadDim;
        const double* kr = Ks + lane * kKsStride;
        double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
#pragma unroll 8
        for (int d = 0; d < kHeadDim; d += 4) {
          a0 = fma(q[d], kr[d], a0);
          a1 = fma(q[d + 1], kr[d + 1], a1);
          a2 = fma(q[d + 2], kr[d + 2], a2);
          a3 = fma(q[d + 3], kr[d + 3], a3);
        }
        row_scores[j] = (a0 + a1) + (a2 + a3);
      }
    }
    __syncthreads();
    // selection: warp per row
    if (i < Nmax) {
      int32_t* out = sel + (bh * Nmax + i) * stride;
      int cnt = 0;
      if (i < n) {
        const int m = min(k, i);
        if (m == i) {
          for (int j = lane; j < i; j += 32) out[j] = j;
          cnt = i;
        } else if (m > 0) {
          cnt = warp_select_topm(row_scores, i, m, hist + warp * 256, out);
        }
        if (lane == 0) out[cnt] = i;
        cnt += 1;
      }
      for (int q = cnt + lane; q < stride; q += 32) out[q] = -1;
      if (lane == 0) n_sel[bh * Nmax + i] = cnt;
    }
    __syncthreads();
  }
}

size_t smem_bytes(int Nmax, bool use_ws) {
  size_t s = sizeof(double) * (kRows * kHeadDim + kJT * kKsStride) + sizeof(int) * kRows * 256;
  if (!use_ws) s += sizeof(double) * (size_t)kRows * Nmax;
  return s;
}

}  // namespace

int score_topk_stride(int k, int Nmax) { return (k < Nmax - 1 ? k : Nmax - 1) + 1; }

size_t score_topk_ws_bytes(int B, int Hq, int Nmax) {
  if (Nmax <= kSmemScoreCap) return 0;
  return sizeof(double) * (size_t)kWsCtas * kRows * Nmax;
}

int launch_score_topk(const float* Qp, const float* Kp, int B, int Hq, int Hkv, int Nmax, const int32_t* n_chunks,
                      int k, int32_t* sel, int32_t* n_sel, void* ws, cudaStream_t stream) {
  const bool use_ws = Nmax > kSmemScoreCap;
  const long long n_blocks = (long long)B * Hq * ((Nmax + kRows - 1) / kRows);
  const size_t smem = smem_bytes(Nmax, use_ws);
  cudaError_t e = cudaFuncSetAttribute(score_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return cuda_status(e);
  long long grid = use_ws ? (n_blocks < kWsCtas ? n_blocks : kWsCtas) : n_blocks;
  if (grid > 0x7fffffffLL) grid = 0x7fffffffLL;
  score_topk_kernel<<<(unsigned)grid, 256, smem, stream>>>(Qp, Kp, Hq, Hq / Hkv, Nmax, n_chunks, k,
                                                            score_topk_stride(k, Nmax), sel, n_sel, n_blocks,
                                                            use_ws ? static_cast<double*>(ws) : nullptr);
  return launch_status();
}

}  // namespace dhsa

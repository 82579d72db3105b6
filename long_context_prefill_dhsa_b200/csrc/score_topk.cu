// Chunk similarity + causal per-query-chunk top-k (stages 2-3 of the DHSA routing).
//
// gist.science technical summary of "Long-Context Modeling with Dynamic
// Hierarchical Sparse Attention", "Hierarchical Routing Formulation": a
// chunk-level similarity matrix scores chunk-to-chunk interactions (Step 1)
// and each query chunk is routed to a compact set of key chunks under the
// causal constraint (Step 2). Here: S[i][j] = <Qp_i, Kp_j> for j < i, and the
// kept set is {i} + the min(k, i) earlier chunks ranked by (S desc, j asc).
//
// The ranking is decided on the fp64 dot products of the fp32 pooled vectors
// (fp32 x fp32 products are exact in fp64), but only a handful of scores per
// row are ever computed in fp64:
//   1. score kernel: fp32 FFMA scores of 64-row x 128-key tiles of the lower
//      triangle (register-tiled, both operands staged in shared memory),
//      stored packed per row (row i holds its i scores) in the workspace;
//      some of its tiles also write ||Kp_j||_2 of every pooled key row
//      (rounded up).
//   2. select kernel, one warp per row (its scores staged once in shared
//      memory when the row has at most 1024): a radix select in digits of
//      8 bits over the order-preserving fp32 keys, from the highest bit in
//      which the row's keys differ, finds the m-th largest fp32 score T. The
//      fp32 dot product of n = 128 terms is within gamma_n * ||q|| * ||k||
//      of the exact one (gamma_n = n u / (1 - n u), u = 2^-24), so with D
//      = 2 gamma_n ||q_i|| max_j ||k_j|| every score above T + D is in the
//      exact top-m and every score below T - D is out. Only the band
//      [T - D, T + D] is re-scored in fp64 and ranked exactly (ties to the
//      lower index). The kept indices are written ascending, diagonal last.
// For very many chunks the workspace is processed in batches of heads.
#include "common.cuh"
#include "pool_row.cuh"
#include "sm100_ptx.cuh"

namespace dhsa {
namespace {

constexpr int TR = 64;            // query rows per score tile
constexpr int TK = 128;           // keys per score tile
constexpr int kKsStride = kHeadDim + 4;
constexpr size_t kWsCap = size_t(256) << 20;   // scores of one head batch
constexpr double kU = 5.9604644775390625e-08;   // 2^-24
constexpr double kGamma = 128.0 * kU / (1.0 - 128.0 * kU);
constexpr int kBudgetCap = 256;   // a budget row keeps at most kBudgetCap - 1 earlier chunks

__device__ __forceinline__ unsigned order_key32(float s) {
  const unsigned u = __float_as_uint(s);
  return (u >> 31) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

__host__ __device__ __forceinline__ long long tri(long long i) { return i * (i - 1) / 2; }

// Loads of the pooled vectors, key norms and scores. The separate kernels read
// buffers an earlier launch wrote and use plain loads; the fused routing
// kernel reads buffers other blocks of the same launch wrote (after a grid
// barrier), so its instantiation (kCoh) loads through L2 (ld.global.cg),
// never through a possibly stale or non-coherent L1 line.
template <bool kCoh>
__device__ __forceinline__ float ldf(const float* p) {
  if constexpr (kCoh) return __ldcg(p);
  else return *p;
}
template <bool kCoh>
__device__ __forceinline__ float4 ldf4(const float* p) {
  if constexpr (kCoh) return __ldcg(reinterpret_cast<const float4*>(p));
  else return *reinterpret_cast<const float4*>(p);
}

// ------------------------------------------------------------------ 1. key norms
// one warp: the norm of a 128-float row whose lane-th float4 is v (every
// lane gets it); the fixed order makes every caller bit-identical
__device__ __forceinline__ float warp_row_norm(const float4 v) {
  double s = (double)v.x * v.x + (double)v.y * v.y + (double)v.z * v.z + (double)v.w * v.w;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  return (float)(sqrt(s) * (1.0 + 1e-6));   // fp32 rounding covered by the margin
}

// one warp: the norm of pooled key row r
template <bool kCoh>
__device__ __forceinline__ void key_norm_row(const float* __restrict__ Kp, long long r, float* __restrict__ kn) {
  const int lane = threadIdx.x & 31;
  const float nrm = warp_row_norm(ldf4<kCoh>(Kp + r * kHeadDim + 4 * lane));
  if (lane == 0) kn[r] = nrm;
}

// ------------------------------------------------------------------ 2. fp32 score tiles
// one block: score tile (rb, kb) of head bh0 + bhl into that head's packed
// rows of ws; a tile is TR query rows x 32 * KC keys (sm: TR * 128 +
// 32 * KC * 132 floats of shared memory). Every score is one thread's fp32
// dot product in a fixed order, whatever KC. With kn given, the tiles of the
// last row block of each kv group's first query head also write the norms
// of their keys (computed from the staged rows exactly as key_norm_row does):
// those tiles cover every key some row scores, once per kv head.
template <int KC, bool kCoh>
__device__ __forceinline__ void score_tile_body(const float* __restrict__ Qp, const float* __restrict__ Kp, int Hq,
                                                int G, int Nmax, const int32_t* __restrict__ n_chunks, long long bh0,
                                                int bhl, int rb, int kb, float* __restrict__ ws, float* sm,
                                                float* __restrict__ kn = nullptr) {
  float* Qs = sm;                        // [TR][128]
  float* Ks = sm + TR * kHeadDim;        // [32 * KC][132]
  const long long bh = bh0 + bhl;
  const int b = (int)(bh / Hq), hq = (int)(bh % Hq);
  const int n = min(max(n_chunks[b], 0), Nmax);   // a count outside [0, Nmax] is clamped
  const int i0 = rb * TR, j0 = kb * 32 * KC;
  const int i_hi = min(i0 + TR, n);                 // rows [i0, i_hi)
  if (i0 >= n || j0 >= i_hi - 1) return;            // no j < i in this tile
  const long long kv_row0 = ((long long)b * (Hq / G) + hq / G) * Nmax;
  for (int idx = threadIdx.x; idx < TR * 32; idx += blockDim.x) {
    const int r = idx >> 5, c4 = idx & 31;
    const int i = i0 + r;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (i < n) v = ldf4<kCoh>(Qp + (bh * Nmax + i) * kHeadDim + 4 * c4);
    reinterpret_cast<float4*>(Qs + r * kHeadDim)[c4] = v;
  }
  for (int idx = threadIdx.x; idx < 32 * KC * 32; idx += blockDim.x) {
    const int r = idx >> 5, c4 = idx & 31;
    const int j = j0 + r;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (j < n) v = ldf4<kCoh>(Kp + (kv_row0 + j) * kHeadDim + 4 * c4);
    reinterpret_cast<float4*>(Ks + r * kKsStride)[c4] = v;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (kn && hq % G == 0 && rb == (n - 1) / TR) {
    for (int r = warp; r < 32 * KC && j0 + r < n; r += 8) {
      const float nrm = warp_row_norm(*reinterpret_cast<const float4*>(Ks + r * kKsStride + 4 * lane));
      if (lane == 0) kn[kv_row0 + j0 + r] = nrm;
    }
  }
  float acc[8][KC];
#pragma unroll
  for (int r = 0; r < 8; ++r)
#pragma unroll
    for (int c = 0; c < KC; ++c) acc[r][c] = 0.f;
#pragma unroll 2
  for (int d = 0; d < kHeadDim; d += 4) {
    float4 kv[KC];
#pragma unroll
    for (int c = 0; c < KC; ++c) kv[c] = *reinterpret_cast<const float4*>(Ks + (lane + 32 * c) * kKsStride + d);
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const float4 qv = *reinterpret_cast<const float4*>(Qs + (warp * 8 + r) * kHeadDim + d);
#pragma unroll
      for (int c = 0; c < KC; ++c) {
        acc[r][c] = fmaf(qv.x, kv[c].x, acc[r][c]);
        acc[r][c] = fmaf(qv.y, kv[c].y, acc[r][c]);
        acc[r][c] = fmaf(qv.z, kv[c].z, acc[r][c]);
        acc[r][c] = fmaf(qv.w, kv[c].w, acc[r][c]);
      }
    }
  }
  float* head = ws + bhl * tri(Nmax);
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    const int i = i0 + warp * 8 + r;
    if (i >= i_hi) continue;
#pragma unroll
    for (int c = 0; c < KC; ++c) {
      const int j = j0 + lane + 32 * c;
      if (j < i) head[tri(i) + j] = acc[r][c];
    }
  }
}

__global__ void __launch_bounds__(256, 2) score_tile_kernel(const float* __restrict__ Qp,
                                                         const float* __restrict__ Kp, int Hq, int G, int Nmax,
                                                         const int32_t* __restrict__ n_chunks, long long bh0,
                                                         int n_rb, int n_kb, float* __restrict__ ws,
                                                         float* __restrict__ kn) {
  extern __shared__ __align__(16) float sm[];
  score_tile_body<TK / 32, false>(Qp, Kp, Hq, G, Nmax, n_chunks, bh0, blockIdx.y, blockIdx.x / n_kb, blockIdx.x % n_kb, ws,
                                  sm, kn);
}

// ------------------------------------------------------------------ 3. selection
template <bool kCoh>
__device__ double exact_score(const float* __restrict__ q, const float* __restrict__ k) {
  double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
  // unrolled so that the loads of several steps are in flight together (the
  // rows come from L2; a rolled loop waits for each pair in turn)
#pragma unroll 8
  for (int d = 0; d < kHeadDim; d += 4) {
    const float4 x = ldf4<kCoh>(q + d);
    const float4 y = ldf4<kCoh>(k + d);
    a0 = fma((double)x.x, (double)y.x, a0);
    a1 = fma((double)x.y, (double)y.y, a1);
    a2 = fma((double)x.z, (double)y.z, a2);
    a3 = fma((double)x.w, (double)y.w, a3);
  }
  return (a0 + a1) + (a2 + a3);
}

// (score desc, index asc) as one comparison: does (sa, ja) rank above (sb, jb)?
__device__ __forceinline__ bool ranks_above(double sa, int ja, double sb, int jb) {
  return sa > sb || (sa == sb && ja < jb);
}

// The exact top-m of candidates j < c of one row, m < c, as a cut: scores
// above hi are in, below lo are out, and a band score is in iff it does not
// rank below (cutE, cutJ) (or the whole band is in). Executed by one warp;
// `hist` is that warp's 256-int shared scratch.
struct Cut {
  double lo, hi, cutE;
  float lo_f, hi_f;   // the band's bounds rounded inward to fp32: for a float s,
                      // s >= lo iff s >= lo_f and s <= hi iff s <= hi_f
  int cutJ;
  int nlist;          // >= 0: the band members inside the cut are the first nlist
                      // entries of the warp's hist area (no re-scoring needed)
  bool all_band;
};

constexpr int kRowCap = 1024;   // scores of a row a warp stages in shared memory
constexpr int kSelectSmem = 8 * kRowCap * (int)sizeof(float);   // dynamic shared memory of the selection kernels

// A row of packed scores: a warp's copy in shared memory when the row fits
// (every pass of the selection then reads shared memory instead of
// re-reading global memory with dependent loads), else the row in global
// memory.
struct RowSrc {
  const float* p;
  bool smem;
};

template <bool kCoh>
__device__ __forceinline__ float rd(const RowSrc& r, int j) {
  if constexpr (kCoh) {
    if (!r.smem) return __ldcg(r.p + j);
  }
  return r.p[j];
}

// one warp: stage row[0 .. c) into its buffer when it fits
template <bool kCoh>
__device__ __forceinline__ RowSrc stage_row(const float* row, int c, float* buf) {
  if (c > kRowCap) return RowSrc{row, false};
  const int lane = threadIdx.x & 31;
  for (int j0 = 0; j0 < c; j0 += 256) {
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int j = j0 + lane + 32 * u;
      v[u] = j < c ? ldf<kCoh>(row + j) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int j = j0 + lane + 32 * u;
      if (j < c) buf[j] = v[u];
    }
  }
  __syncwarp();
  return RowSrc{buf, true};
}

template <bool kCoh>
__device__ Cut topm_cut(const RowSrc& row, int c, int m, int* hist, const float* __restrict__ qrow,
                        const float* __restrict__ Kp, long long kv_row0, const float* __restrict__ kn) {
  const int lane = threadIdx.x & 31;
  const unsigned full = 0xffffffffu;
  // --- radix select of the m-th largest fp32 key, over the bits in which
  // the row's keys differ: the leading bits all keys share (sign and
  // exponent, mostly) would put every key in one or two bins and serialise
  // the histogram's shared-memory atomics
  unsigned key_hi = 0u, key_lo = 0xffffffffu;
  for (int j = lane; j < c; j += 32) {
    const unsigned kk = order_key32(rd<kCoh>(row, j));
    key_hi = max(key_hi, kk);
    key_lo = min(key_lo, kk);
  }
  key_hi = __reduce_max_sync(full, key_hi);
  key_lo = __reduce_min_sync(full, key_lo);
  const unsigned diff = key_hi ^ key_lo;
  int hi = diff ? 31 - __clz(diff) : -1;      // highest bit still to resolve
  unsigned mask = diff ? ~((2u << hi) - 1u) : 0xffffffffu;
  unsigned prefix = key_hi & mask;            // every key equal: the m-th largest is that key
  int need = m;
  while (hi >= 0) {
    const int shift = hi >= 7 ? hi - 7 : 0;
    const unsigned dmask = (2u << (hi - shift)) - 1u;   // a digit of at most 8 bits
    for (int q = lane; q < 256; q += 32) hist[q] = 0;
    __syncwarp();
    for (int j = lane; j < c; j += 32) {
      const unsigned kk = order_key32(rd<kCoh>(row, j));
      if ((kk & mask) == prefix) atomicAdd(&hist[(kk >> shift) & dmask], 1);
    }
    __syncwarp();
    int cq[8], lsum = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      cq[q] = hist[255 - 8 * lane - q];
      lsum += cq[q];
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
    int digit = 0, above = 0, inbin = 0;
    if (lane == src) {
      int run = excl;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (run + cq[q] >= need) {
          digit = 255 - 8 * lane - q;
          above = run;
          inbin = cq[q];
          break;
        }
        run += cq[q];
      }
    }
    digit = __shfl_sync(full, digit, src);
    above = __shfl_sync(full, above, src);
    inbin = __shfl_sync(full, inbin, src);
    prefix |= (unsigned)digit << shift;
    mask |= dmask << shift;
    need -= above;
    hi = shift - 1;
    __syncwarp();
    if (hi >= 0 && inbin <= 32) {
      // at most 32 keys share the prefix: gather them (one per lane), sort
      // them descending and take the need-th; no further histogram passes
      int base = 0;
      for (int j0 = 0; j0 < c; j0 += 32) {
        const int j = j0 + lane;
        unsigned kk = 0;
        bool hit = false;
        if (j < c) {
          kk = order_key32(rd<kCoh>(row, j));
          hit = (kk & mask) == prefix;
        }
        const unsigned bb = __ballot_sync(full, hit);
        if (hit) hist[base + __popc(bb & lanemask_lt())] = (int)kk;
        base += __popc(bb);
      }
      __syncwarp();
      unsigned key = lane < inbin ? (unsigned)hist[lane] : 0u;
#pragma unroll
      for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
        for (int stride2 = size >> 1; stride2 > 0; stride2 >>= 1) {
          const unsigned other = __shfl_xor_sync(full, key, stride2);
          const bool up = ((lane & size) == 0);        // this block sorts descending
          const bool lower = ((lane & stride2) == 0);
          key = (lower == up) ? max(key, other) : min(key, other);
        }
      }
      prefix = __shfl_sync(full, key, need - 1);
      hi = -1;
      __syncwarp();
    }
  }
  const unsigned tu = (prefix & 0x80000000u) ? (prefix & 0x7fffffffu) : ~prefix;
  const double T = (double)__uint_as_float(tu);
  // --- rounding band
  const float4 qv = ldf4<kCoh>(qrow + 4 * lane);
  double qq = (double)qv.x * qv.x + (double)qv.y * qv.y + (double)qv.z * qv.z + (double)qv.w * qv.w;
  float kmax = 0.f;
#pragma unroll 4
  for (int j = lane; j < c; j += 32) kmax = fmaxf(kmax, ldf<kCoh>(kn + kv_row0 + j));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    qq += __shfl_xor_sync(full, qq, o);
    kmax = fmaxf(kmax, __shfl_xor_sync(full, kmax, o));
  }
  const double D = 2.0 * kGamma * sqrt(qq) * (1.0 + 1e-6) * (double)kmax;
  Cut cut;
  cut.lo = T - D;
  cut.hi = T + D;
  cut.lo_f = __double2float_ru(cut.lo);
  cut.hi_f = __double2float_rd(cut.hi);
  cut.cutE = -INFINITY;
  cut.cutJ = 0x7fffffff;
  cut.nlist = -1;
  // one pass: count the scores above the band, and list the band's members
  // (their first 256 indices, through the free histogram area)
  int a = 0, nc = 0;
  for (int j0 = 0; j0 < c; j0 += 32) {
    const int j = j0 + lane;
    bool inb = false, abv = false;
    if (j < c) {
      const float s = rd<kCoh>(row, j);
      abv = s > cut.hi_f;
      inb = s >= cut.lo_f && s <= cut.hi_f;
    }
    const unsigned bb = __ballot_sync(full, inb);
    const int pos = nc + __popc(bb & lanemask_lt());
    if (inb && pos < 256) hist[pos] = j;
    nc += __popc(bb);
    a += __popc(__ballot_sync(full, abv));
  }
  __syncwarp();
  const int r = m - a;              // 1 <= r <= nc
  // --- exact cut (E*, j*) among the band: the r-th by (exact desc, j asc)
  cut.all_band = (r >= nc);
  if (cut.all_band) return cut;
  if (nc <= 32) {
    // the band sits in lanes 0..nc-1: score exactly, bitonic sort best-first
    const int my_j = lane < nc ? hist[lane] : -1;
    __syncwarp();
    double my_e = -INFINITY;
    int my_key_j = 0x7fffffff;
    if (my_j >= 0) {
      my_e = exact_score<kCoh>(qrow, Kp + (kv_row0 + my_j) * kHeadDim);
      my_key_j = my_j;
    }
#pragma unroll
    for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
      for (int stride2 = size >> 1; stride2 > 0; stride2 >>= 1) {
        const double oe = __shfl_xor_sync(full, my_e, stride2);
        const int oj = __shfl_xor_sync(full, my_key_j, stride2);
        const bool up = ((lane & size) == 0);          // this block sorts best-first
        const bool lower = ((lane & stride2) == 0);
        const bool mine_above = ranks_above(my_e, my_key_j, oe, oj);
        const bool keep_mine = (lower == up) ? mine_above : !mine_above;
        if (!keep_mine) {
          my_e = oe;
          my_key_j = oj;
        }
      }
    }
    cut.cutE = __shfl_sync(full, my_e, r - 1);
    cut.cutJ = __shfl_sync(full, my_key_j, r - 1);
    // the r best band members (lanes 0 .. r-1 after the sort), for in_cut
    if (lane < r) hist[lane] = my_key_j;
    __syncwarp();
    cut.nlist = r;
  } else {
    // many candidates (heavy ties): r rounds of "best below the previous pick"
    double pe = INFINITY;
    int pj = -1;
    for (int t = 0; t < r; ++t) {
      double be = -INFINITY;
      int bj = 0x7fffffff;
      for (int j = lane; j < c; j += 32) {
        const float s = rd<kCoh>(row, j);
        if (s < cut.lo_f || s > cut.hi_f) continue;
        const double e = exact_score<kCoh>(qrow, Kp + (kv_row0 + j) * kHeadDim);
        if (ranks_above(pe, pj, e, j) && ranks_above(e, j, be, bj)) {
          be = e;
          bj = j;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const double oe = __shfl_xor_sync(full, be, o);
        const int oj = __shfl_xor_sync(full, bj, o);
        if (ranks_above(oe, oj, be, bj)) {
          be = oe;
          bj = oj;
        }
      }
      pe = be;
      pj = bj;
    }
    cut.cutE = pe;
    cut.cutJ = pj;
  }
  return cut;
}

// Is candidate j (fp32 score s) inside the exact top-m described by `cut`?
// (list: the warp's hist area, holding the cut's band members when listed)
template <bool kCoh>
__device__ __forceinline__ bool in_cut(const Cut& cut, float s32, int j, const float* __restrict__ qrow,
                                       const float* __restrict__ Kp, long long kv_row0, const int* list) {
  if (s32 > cut.hi_f) return true;
  if (s32 < cut.lo_f) return false;
  if (cut.all_band) return true;
  if (cut.nlist >= 0) {
    for (int t = 0; t < cut.nlist; ++t)
      if (list[t] == j) return true;
    return false;
  }
  return !ranks_above(cut.cutE, cut.cutJ, exact_score<kCoh>(qrow, Kp + (kv_row0 + j) * kHeadDim), j);
}

// one warp: the top-k row wr of the head batch starting at head bh0 (hist:
// this warp's 256 ints of shared scratch)
template <bool kCoh>
__device__ __forceinline__ void select_row(const float* __restrict__ Qp, const float* __restrict__ Kp,
                                           const float* __restrict__ kn, int Hq, int G, int Nmax,
                                           const int32_t* __restrict__ n_chunks, int k, int stride, long long bh0,
                                           long long wr, const float* __restrict__ ws, int32_t* __restrict__ sel,
                                           int32_t* __restrict__ n_sel, int* hist, float* rowbuf) {
  const int lane = threadIdx.x & 31;
  const unsigned full = 0xffffffffu;
  const long long bhl = wr / Nmax;
  const int i = (int)(wr % Nmax);
  const long long bh = bh0 + bhl;
  const int b = (int)(bh / Hq), hq = (int)(bh % Hq);
  const int n = min(max(n_chunks[b], 0), Nmax);   // a count outside [0, Nmax] is clamped
  int32_t* out = sel + (bh * Nmax + i) * stride;
  int cnt = 0;
  if (i < n) {
    const int m = min(k, i);
    if (m == i) {
      for (int j = lane; j < i; j += 32) out[j] = j;
      cnt = i;
    } else if (m > 0) {
      const RowSrc row = stage_row<kCoh>(ws + bhl * tri(Nmax) + tri(i), i, rowbuf);
      const long long kv_row0 = ((long long)b * (Hq / G) + hq / G) * Nmax;
      const float* qrow = Qp + (bh * Nmax + i) * kHeadDim;
      const Cut cut = topm_cut<kCoh>(row, i, m, hist, qrow, Kp, kv_row0, kn);
      // --- output, ascending
      int written = 0;
      for (int j0 = 0; j0 < i; j0 += 32) {
        const int j = j0 + lane;
        const bool take = j < i && in_cut<kCoh>(cut, rd<kCoh>(row, j), j, qrow, Kp, kv_row0, hist);
        const unsigned bt = __ballot_sync(full, take);
        const int pos = written + __popc(bt & lanemask_lt());
        if (take && pos < m) out[pos] = j;
        written += __popc(bt);
      }
      cnt = written < m ? written : m;
    }
    if (lane == 0) out[cnt] = i;
    cnt += 1;
  }
  for (int q = cnt + lane; q < stride; q += 32) out[q] = -1;
  if (lane == 0) n_sel[bh * Nmax + i] = cnt;
}

// sum_{i < n} min(kk, i)
__device__ __forceinline__ long long topk_prefix(long long n, long long kk) {
  return n <= kk + 1 ? n * (n - 1) / 2 : kk * (kk + 1) / 2 + kk * (n - kk - 1);
}

// Block CSR of the top-k rule written straight from the selection. Under
// that rule row i < n_b keeps min(k, i) + 1 chunks, so the CSR offset of a
// row has a closed form: the rows before (b, hq, i) hold the sum over earlier
// batch elements b' of Hq T(n_b'), plus hq T(n_b), plus i + F(i), with
// F(i) = sum_{i' < i} min(k, i') and T(n) = n + F(n). Results equal the scan
// and fill of csr.cu, bit for bit.
// one warp: the CSR row of (bh, i) from its selection row (just written by
// this warp; n_sel[bh * Nmax + i] holds its length)
__device__ void csr_row(const CsrOut& o, const int32_t* sel, const int32_t* n_sel, const int32_t* n_chunks, int B,
                        int Hq, int Nmax, int stride, long long bh, int i) {
  const int lane = threadIdx.x & 31;
  const int b = (int)(bh / Hq), hq = (int)(bh % Hq);
  const long long kk = stride - 1;
  long long base = 0;
  for (int bb = 0; bb < b; ++bb) {
    const long long nb = min(max(n_chunks[bb], 0), Nmax);
    base += (long long)Hq * (nb + topk_prefix(nb, kk));
  }
  const long long n = min(max(n_chunks[b], 0), Nmax);
  const long long T = n + topk_prefix(n, kk);
  base += hq * T;
  const long long rp = i < n ? base + i + topk_prefix(i, kk) : base + T;
  const long long r = bh * Nmax + i;
  const int cnt = __ldcg(n_sel + r);   // written by this warp in this launch: read through L2
  const int want = i < n ? (int)min((long long)i, kk) + 1 : 0;
  const int32_t* src = sel + r * stride;
  const int32_t* ob = o.off + (long long)b * (Nmax + 1);
  long long keys = 0;
  for (int q = lane; q < want; q += 32) {
    const int j = q < cnt ? __ldcg(src + q) : i;
    o.col_idx[rp + q] = j;
    keys += ob[j + 1] - ob[j];
  }
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) keys += __shfl_xor_sync(0xffffffffu, keys, s);
  if (lane == 0) {
    if (cnt != want) raise_device_flag(o.status, DHSA_DEVFLAG_BAD_SELECTION);
    o.row_ptr[r] = (int32_t)rp;
    if (r == (long long)B * Hq * Nmax - 1) o.row_ptr[r + 1] = (int32_t)(rp + want);
    if (o.cost) o.cost[r] = i < n ? (long long)(ob[i + 1] - ob[i]) * keys : 0;
  }
}

__global__ void __launch_bounds__(256) select_kernel(const float* __restrict__ Qp, const float* __restrict__ Kp,
                                                     const float* __restrict__ kn, int Hq, int G, int Nmax,
                                                     const int32_t* __restrict__ n_chunks, int k, int stride,
                                                     long long bh0, long long n_rows,
                                                     const float* __restrict__ ws, int32_t* sel, int32_t* n_sel,
                                                     int B, CsrOut csr) {
  __shared__ int hist_all[8][256];
  extern __shared__ __align__(16) float rowbuf_all[];   // [8][kRowCap]
  const int warp = threadIdx.x >> 5;
  const long long wr = (long long)blockIdx.x * 8 + warp;      // row within the head batch
  if (wr >= n_rows) return;
  select_row<false>(Qp, Kp, kn, Hq, G, Nmax, n_chunks, k, stride, bh0, wr, ws, sel, n_sel, hist_all[warp],
                    rowbuf_all + warp * kRowCap);
  if (csr.row_ptr) {
    __syncwarp();
    csr_row(csr, sel, n_sel, n_chunks, B, Hq, Nmax, stride, bh0 + wr / Nmax, (int)(wr % Nmax));
  }
}

// ------------------------------------------------------------------ 3'. row budgets
// README, "Predictor Checkpoints": fixed or query-dependent row budgets;
// gist.science technical summary, "Significance and Claims": N_b is the token
// budget. A row keeps its diagonal chunk, the r = min(recent, i, k_max)
// chunks just before it, then earlier chunks j < i - r by (score desc,
// index asc) while the kept earlier tokens are fewer than its budget, at
// most k_max earlier chunks in all. Only the top m = min(k_max - r, i - r)
// ranked candidates can be taken: their set comes from the same exact cut
// as the top-k rule, then they are re-scored in fp64, ranked, and the
// budget is applied along that order.
__global__ void __launch_bounds__(256) budget_select_kernel(
    const float* __restrict__ Qp, const float* __restrict__ Kp, const float* __restrict__ kn, int Hq, int G,
    int Nmax, const int32_t* __restrict__ n_chunks, const int32_t* __restrict__ off, int budget,
    const int32_t* __restrict__ budgets, int recent, int k_max, int stride, long long bh0, long long n_rows,
    const float* __restrict__ ws, int32_t* __restrict__ sel, int32_t* __restrict__ n_sel) {
  __shared__ int hist_all[8][256];
  __shared__ int mj_all[8][kBudgetCap];      // members, ascending index
  __shared__ double me_all[8][kBudgetCap];   // their exact scores
  __shared__ int ml_all[8][kBudgetCap];      // chunk lengths by rank
  extern __shared__ __align__(16) float rowbuf_all[];   // [8][kRowCap]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const unsigned full = 0xffffffffu;
  const long long wr = (long long)blockIdx.x * 8 + warp;
  if (wr >= n_rows) return;
  const long long bhl = wr / Nmax;
  const int i = (int)(wr % Nmax);
  const long long bh = bh0 + bhl;
  const int b = (int)(bh / Hq), hq = (int)(bh % Hq);
  const int n = min(max(n_chunks[b], 0), Nmax);   // a count outside [0, Nmax] is clamped
  int32_t* out = sel + (bh * Nmax + i) * stride;
  int* hist = hist_all[warp];
  int* mj = mj_all[warp];
  double* me = me_all[warp];
  int* ml = ml_all[warp];
  int cnt = 0;
  if (i < n) {
    const int32_t* ob = off + (long long)b * (Nmax + 1);
    const int r = min(min(recent, i), k_max);
    const int c = i - r;                           // ranked candidates j < c
    const int m = min(k_max - r, c);
    const long long used0 = (long long)ob[i] - ob[i - r];
    const long long bud = budgets ? (long long)budgets[bh * Nmax + i] : (long long)budget;
    int t = 0;
    if (m > 0 && used0 < bud) {
      const RowSrc row = stage_row<false>(ws + bhl * tri(Nmax) + tri(i), c, rowbuf_all + warp * kRowCap);
      const long long kv_row0 = ((long long)b * (Hq / G) + hq / G) * Nmax;
      const float* qrow = Qp + (bh * Nmax + i) * kHeadDim;
      const bool all = (m == c);
      Cut cut{};
      if (!all) cut = topm_cut<false>(row, c, m, hist, qrow, Kp, kv_row0, kn);
      // members of the top m, ascending index
      int nm = 0;
      for (int j0 = 0; j0 < c; j0 += 32) {
        const int j = j0 + lane;
        const bool take = j < c && (all || in_cut<false>(cut, rd<false>(row, j), j, qrow, Kp, kv_row0, hist));
        const unsigned bt = __ballot_sync(full, take);
        const int pos = nm + __popc(bt & lanemask_lt());
        if (take && pos < m) mj[pos] = j;
        nm += __popc(bt);
      }
      nm = min(nm, m);
      __syncwarp();
      for (int a = lane; a < nm; a += 32) me[a] = exact_score<false>(qrow, Kp + (kv_row0 + mj[a]) * kHeadDim);
      __syncwarp();
      // rank of each member; lengths in rank order
      for (int a = lane; a < nm; a += 32) {
        const double ea = me[a];
        const int ja = mj[a];
        int rank = 0;
        for (int q = 0; q < nm; ++q) rank += ranks_above(me[q], mj[q], ea, ja);
        hist[a] = rank;
        ml[rank] = ob[ja + 1] - ob[ja];
      }
      __syncwarp();
      // ranks 0..t-1 are taken: those reached while the kept tokens are below the budget
      long long run = used0;
      for (int q0 = 0; q0 < nm; q0 += 32) {
        const int q = q0 + lane;
        const int v = q < nm ? ml[q] : 0;
        int incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int u = __shfl_up_sync(full, incl, o);
          if (lane >= o) incl += u;
        }
        t += __popc(__ballot_sync(full, q < nm && run + (incl - v) < bud));
        run += __shfl_sync(full, incl, 31);
      }
      // taken members, ascending
      int written = 0;
      for (int a0 = 0; a0 < nm; a0 += 32) {
        const int a = a0 + lane;
        const bool take = a < nm && hist[a] < t;
        const unsigned bt = __ballot_sync(full, take);
        if (take) out[written + __popc(bt & lanemask_lt())] = mj[a];
        written += __popc(bt);
      }
    }
    cnt = t;
    for (int q = lane; q < r; q += 32) out[cnt + q] = i - r + q;   // the recent window
    cnt += r;
    if (lane == 0) out[cnt] = i;
    cnt += 1;
  }
  for (int q = cnt + lane; q < stride; q += 32) out[q] = -1;
  if (lane == 0) n_sel[bh * Nmax + i] = cnt;
}

long long heads_per_batch(int B, int Hq, int Nmax) {
  const size_t per_head = sizeof(float) * (size_t)tri(Nmax);
  long long h = per_head ? (long long)(kWsCap / per_head) : (long long)B * Hq;
  if (h < 1) h = 1;
  if (h > (long long)B * Hq) h = (long long)B * Hq;
  if (h > 65535) h = 65535;   // grid.y limit
  return h;
}


// ------------------------------------------------------------------ 4. fused routing
// Pooling of Q and K, key norms, score tiles, the top-k selection and (when
// asked) the block CSR in one cooperative launch, with a grid-wide barrier
// between the phases that read what the previous one wrote. Each phase runs
// the same per-warp or per-block code as its separate kernel, so the
// results are bit-identical.
struct GridBar {
  unsigned int* count;    // arrivals so far (zeroed before the launch)
  unsigned int* abort;    // set by a block that gave up waiting (zeroed before the launch)
  unsigned int* status;
  unsigned long long limit_ns;   // wall-clock limit of one barrier wait
  unsigned long long hold_ns;    // test hook: block 0 arrives this late at the first barrier (0: off)
};

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned int* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Every block arrives once per barrier; thread 0 waits until all have. A wait
// that passes limit_ns raises DHSA_DEVFLAG_WAIT_TIMEOUT and the abort word;
// a block that sees the abort word stops waiting. Either way the barrier
// returns false and the block leaves the kernel (the phases after it would
// read unfinished results). Returns true once every block has arrived.
__device__ __forceinline__ bool grid_barrier(const GridBar& gb, unsigned& phase) {
  __shared__ int s_ok;
  __syncthreads();
  ++phase;
  if (threadIdx.x == 0) {
    int ok = 1;
    if (gb.hold_ns && phase == 1 && blockIdx.x == 0) {
      // test hook: arrive late (bounded), or as soon as another block gave up
      const uint64_t t0 = ptx::globaltimer_ns();
      while (ptx::globaltimer_ns() - t0 < gb.hold_ns && ld_acquire_u32(gb.abort) == 0u) __nanosleep(256);
    }
    __threadfence();
    atomicAdd(gb.count, 1u);
    const unsigned target = phase * gridDim.x;
    const uint64_t t0 = ptx::globaltimer_ns();
    while (ld_acquire_u32(gb.count) < target) {
      if (ld_acquire_u32(gb.abort) != 0u) {
        ok = 0;
        break;
      }
      if (ptx::globaltimer_ns() - t0 > gb.limit_ns) {
        atomicExch(gb.abort, 1u);
        raise_device_flag(gb.status, DHSA_DEVFLAG_WAIT_TIMEOUT);
        ok = 0;
        break;
      }
      __nanosleep(64);
    }
    __threadfence();
    s_ok = ok;
  }
  __syncthreads();
  return s_ok != 0;
}

constexpr int kFusedKC = 2;   // 64-key score tiles in the fused kernel: three blocks per SM

__global__ void __launch_bounds__(256, 3) route_fused_kernel(const uint4* __restrict__ Q, const uint4* __restrict__ K,
                                                          int B, int Hq, int Hkv, int L,
                                                          const int32_t* __restrict__ off,
                                                          const int32_t* __restrict__ n_chunks, int Nmax, int k,
                                                          int stride, long long hb, float* __restrict__ Qp,
                                                          float* __restrict__ Kp, float* __restrict__ kn,
                                                          float* __restrict__ scores, int32_t* sel, int32_t* n_sel,
                                                          GridBar gb, CsrOut csr) {
  extern __shared__ __align__(16) float sm[];
  const int G = Hq / Hkv;
  const long long gwarp = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = (long long)gridDim.x * (blockDim.x >> 5);
  unsigned phase = 0;
  // pooled Q and K rows
  const long long rows_q = (long long)B * Hq * Nmax, rows_k = (long long)B * Hkv * Nmax;
  for (long long w = gwarp; w < rows_q + rows_k; w += nwarps) {
    if (w < rows_q) pool_row(Q, Hq, L, off, n_chunks, Nmax, w, Qp, gb.status);
    else pool_row(K, Hkv, L, off, n_chunks, Nmax, w - rows_q, Kp, gb.status);
  }
  if (!grid_barrier(gb, phase)) return;
  // key norms (read by the selection only) and the score tiles of each head batch
  for (long long r = gwarp; r < rows_k; r += nwarps) key_norm_row<true>(Kp, r, kn);
  const int n_rb = (Nmax + TR - 1) / TR, n_kb = (Nmax + 32 * kFusedKC - 1) / (32 * kFusedKC);
  const long long total = (long long)B * Hq;
  int* hist = reinterpret_cast<int*>(sm) + (threadIdx.x >> 5) * 256;
  float* rowbuf = sm + 8 * 256 + (threadIdx.x >> 5) * kRowCap;   // fits in the score tiles' shared memory
  for (long long h0 = 0; h0 < total; h0 += hb) {
    const long long nh = total - h0 < hb ? total - h0 : hb;
    const long long tiles = nh * n_rb * n_kb;
    for (long long t = blockIdx.x; t < tiles; t += gridDim.x) {
      const int bhl = (int)(t / (n_rb * n_kb)), rest = (int)(t % (n_rb * n_kb));
      score_tile_body<kFusedKC, true>(Qp, Kp, Hq, G, Nmax, n_chunks, h0, bhl, rest / n_kb, rest % n_kb, scores, sm);
      __syncthreads();   // the next tile restages shared memory
    }
    if (!grid_barrier(gb, phase)) return;
    for (long long wr = gwarp; wr < nh * Nmax; wr += nwarps) {
      select_row<true>(Qp, Kp, kn, Hq, G, Nmax, n_chunks, k, stride, h0, wr, scores, sel, n_sel, hist, rowbuf);
      if (csr.row_ptr) {
        __syncwarp();
        csr_row(csr, sel, n_sel, n_chunks, B, Hq, Nmax, stride, h0 + wr / Nmax, (int)(wr % Nmax));
      }
    }
    if (h0 + hb < total && !grid_barrier(gb, phase)) return;   // the next head batch overwrites the scores
  }
}

}  // namespace

int score_topk_stride(int k, int Nmax) { return (k < Nmax - 1 ? k : Nmax - 1) + 1; }

size_t score_topk_ws_bytes(int B, int Hq, int Nmax) {
  // key norms (B * Hq rows at most, since Hkv <= Hq) + packed scores of one head batch
  const size_t kn = sizeof(float) * (size_t)B * Hq * Nmax;
  const size_t scores = sizeof(float) * (size_t)tri(Nmax) * heads_per_batch(B, Hq, Nmax);
  return 256 + ((kn + 255) & ~size_t(255)) + scores;
}

int launch_score_topk(const float* Qp, const float* Kp, int B, int Hq, int Hkv, int Nmax, const int32_t* n_chunks,
                      int k, int32_t* sel, int32_t* n_sel, void* ws, const CsrOut& csr, cudaStream_t stream) {
  const int G = Hq / Hkv;
  const int stride = score_topk_stride(k, Nmax);
  float* kn = reinterpret_cast<float*>(static_cast<char*>(ws) + 256);
  const size_t kn_bytes = (sizeof(float) * (size_t)B * Hq * Nmax + 255) & ~size_t(255);
  float* scores = reinterpret_cast<float*>(static_cast<char*>(ws) + 256 + kn_bytes);
  const size_t smem = sizeof(float) * (TR * kHeadDim + TK * kKsStride);
  cudaError_t e = cudaFuncSetAttribute(score_tile_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSelectSmem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(budget_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSelectSmem);
  if (e != cudaSuccess) return cuda_status(e);
  int st = DHSA_OK;
  const int n_rb = (Nmax + TR - 1) / TR, n_kb = (Nmax + TK - 1) / TK;
  const long long total = (long long)B * Hq, hb = heads_per_batch(B, Hq, Nmax);
  for (long long h0 = 0; h0 < total; h0 += hb) {
    const long long nh = (total - h0 < hb) ? total - h0 : hb;
    dim3 grid((unsigned)(n_rb * n_kb), (unsigned)nh);
    // the score tiles also write the key norms the selection reads
    score_tile_kernel<<<grid, 256, smem, stream>>>(Qp, Kp, Hq, G, Nmax, n_chunks, h0, n_rb, n_kb, scores, kn);
    if ((st = launch_status()) != DHSA_OK) return st;
    const long long rows = nh * Nmax;
    select_kernel<<<(unsigned)((rows + 7) / 8), 256, kSelectSmem, stream>>>(Qp, Kp, kn, Hq, G, Nmax, n_chunks, k, stride, h0,
                                                                  rows, scores, sel, n_sel, B, csr);
    if ((st = launch_status()) != DHSA_OK) return st;
  }
  return DHSA_OK;
}

// All of routing up to the selection (and the CSR when csr.row_ptr is set)
// in one cooperative launch (workspace as for launch_score_topk; its first 8
// bytes hold the grid barrier's counter and abort word). limit_ns bounds
// each barrier wait; hold_ns > 0 is the test hook that makes block 0 arrive
// late at the first barrier.
int launch_route_fused(const void* Q, const void* K, int B, int Hq, int Hkv, int L, const int32_t* off,
                       const int32_t* n_chunks, int Nmax, int k, float* Qp, float* Kp, int32_t* sel, int32_t* n_sel,
                       const CsrOut& csr, void* ws, unsigned int* status, unsigned long long limit_ns,
                       unsigned long long hold_ns, cudaStream_t stream) {
  const int stride = score_topk_stride(k, Nmax);
  float* kn = reinterpret_cast<float*>(static_cast<char*>(ws) + 256);
  const size_t kn_bytes = (sizeof(float) * (size_t)B * Hq * Nmax + 255) & ~size_t(255);
  float* scores = reinterpret_cast<float*>(static_cast<char*>(ws) + 256 + kn_bytes);
  const long long hb = heads_per_batch(B, Hq, Nmax);
  const int smem = (int)(sizeof(float) * (TR * kHeadDim + 32 * kFusedKC * kKsStride));
  cudaError_t e = cudaFuncSetAttribute(route_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  int dev = 0, sms = 0, per_sm = 0;
  if (e == cudaSuccess) e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, route_fused_kernel, 256, smem);
  if (e == cudaSuccess) e = cudaMemsetAsync(ws, 0, 2 * sizeof(unsigned int), stream);
  if (e != cudaSuccess) return cuda_status(e);
  if (per_sm < 1) return DHSA_ERR_UNSUPPORTED;
  GridBar gb{static_cast<unsigned int*>(ws), static_cast<unsigned int*>(ws) + 1, status, limit_ns, hold_ns};
  const uint4* q4 = static_cast<const uint4*>(Q);
  const uint4* k4 = static_cast<const uint4*>(K);
  CsrOut c = csr;
  void* args[] = {(void*)&q4,     (void*)&k4,   (void*)&B,     (void*)&Hq,   (void*)&Hkv,   (void*)&L,
                  (void*)&off,    (void*)&n_chunks, (void*)&Nmax, (void*)&k, (void*)&stride, (void*)&hb,
                  (void*)&Qp,     (void*)&Kp,   (void*)&kn,    (void*)&scores, (void*)&sel, (void*)&n_sel,
                  (void*)&gb,     (void*)&c};
  e = cudaLaunchCooperativeKernel((const void*)route_fused_kernel, dim3(per_sm * sms), dim3(256), args, (size_t)smem,
                                  stream);
  return cuda_status(e);
}

int score_budget_max_chunks() { return kBudgetCap - 1; }

int launch_score_budget(const float* Qp, const float* Kp, int B, int Hq, int Hkv, int Nmax, const int32_t* off,
                        const int32_t* n_chunks, int budget, const int32_t* budgets, int recent, int k_max,
                        int32_t* sel, int32_t* n_sel, void* ws, cudaStream_t stream) {
  const int G = Hq / Hkv;
  const int stride = score_topk_stride(k_max, Nmax);
  float* kn = reinterpret_cast<float*>(static_cast<char*>(ws) + 256);
  const size_t kn_bytes = (sizeof(float) * (size_t)B * Hq * Nmax + 255) & ~size_t(255);
  float* scores = reinterpret_cast<float*>(static_cast<char*>(ws) + 256 + kn_bytes);
  const size_t smem = sizeof(float) * (TR * kHeadDim + TK * kKsStride);
  cudaError_t e = cudaFuncSetAttribute(score_tile_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSelectSmem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(budget_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSelectSmem);
  if (e != cudaSuccess) return cuda_status(e);
  int st = DHSA_OK;
  const int n_rb = (Nmax + TR - 1) / TR, n_kb = (Nmax + TK - 1) / TK;
  const long long total = (long long)B * Hq, hb = heads_per_batch(B, Hq, Nmax);
  for (long long h0 = 0; h0 < total; h0 += hb) {
    const long long nh = (total - h0 < hb) ? total - h0 : hb;
    dim3 grid((unsigned)(n_rb * n_kb), (unsigned)nh);
    score_tile_kernel<<<grid, 256, smem, stream>>>(Qp, Kp, Hq, G, Nmax, n_chunks, h0, n_rb, n_kb, scores, kn);
    if ((st = launch_status()) != DHSA_OK) return st;
    const long long rows = nh * Nmax;
    budget_select_kernel<<<(unsigned)((rows + 7) / 8), 256, kSelectSmem, stream>>>(
        Qp, Kp, kn, Hq, G, Nmax, n_chunks, off, budget, budgets, recent, k_max, stride, h0, rows, scores, sel,
        n_sel);
    if ((st = launch_status()) != DHSA_OK) return st;
  }
  return DHSA_OK;
}

}  // namespace dhsa

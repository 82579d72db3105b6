// Work lists of the attention kernels. Every (b, hq, chunk i) row's query
// rows are cut into tiles: 128-row tiles for the long-tile kernel
// (attn_fwd.cu) and tiles of at most 64 rows for the short-tile kernel
// (attn_short.cu). The tile policy decides which kernel takes which rows:
//   0  every tile is a 128-row tile;
//   1  a chunk's last tile goes to the short kernel when it holds at most 64
//      rows (the rest of the chunk stays in 128-row tiles);
//   2  every chunk is cut into 64-row tiles for the short kernel.
#include "common.cuh"
#include "tmap.cuh"

namespace dhsa {

constexpr int kShortRows = 64;

namespace {

// (128-row tiles, short tiles) of a chunk of `len` tokens; the short tiles
// start at row 128 * (long tiles) + 64 * k of the chunk
__device__ __forceinline__ int2 tile_counts(int len, int policy) {
  if (policy == 0) return make_int2(ceil_div(len, kQueryTileRows), 0);
  if (policy == 2) return make_int2(0, ceil_div(len, kShortRows));
  const int nt = ceil_div(len, kQueryTileRows);
  if (nt == 0) return make_int2(0, 0);
  const int tail = len - kQueryTileRows * (nt - 1);
  return tail <= kShortRows ? make_int2(nt - 1, 1) : make_int2(nt, 0);
}

// A batch element's offsets table is consistent when 1 <= n <= Nmax,
// off[0] = 0, off[n] = L and every chunk is non-empty. An inconsistent one
// contributes no items (its tile counts could overrun the lists) and sets
// DHSA_DEVFLAG_BAD_OFFSETS.
__device__ __forceinline__ bool chunk_ok(const int32_t* ob, int c, int n, int L) {
  const int s = ob[c], e = ob[c + 1];
  return s >= 0 && e > s && e <= L && (c > 0 || s == 0) && (c < n - 1 || e == L);
}

// Both lists are ordered (b, kv head, chunk, query head within the group,
// tile), so CTAs running at the same time share the K/V of one kv head in L2.
// One CTA per (query head, batch element) writes that head's items; it
// recomputes the per-chunk tile prefix of its batch element (and the tile
// totals of the earlier ones for its base offsets).
__global__ void __launch_bounds__(1024) build_items_kernel(const int32_t* __restrict__ off,
                                                           const int32_t* __restrict__ n_chunks, int B, int Hq,
                                                           int G, int L, int Nmax, int policy, AttnWork w,
                                                           unsigned int* status) {
  __shared__ int2 warp_sum[32];
  __shared__ int2 carry_s;
  const int t = threadIdx.x, lane = t & 31, wp = t >> 5;
  const int hq = blockIdx.x, b = blockIdx.y;
  const int hkv = hq / G, gq = hq % G;
  auto valid = [&](int bb) -> bool {
    const int n = n_chunks[bb];
    const int32_t* ob = off + (long long)bb * (Nmax + 1);
    bool bad = n < 1 || n > Nmax;
    if (!bad)
      for (int c = t; c < n; c += 1024) bad = bad || !chunk_ok(ob, c, n, L);
    return !__syncthreads_or(bad);
  };
  auto totals_of = [&](int bb) -> int2 {   // (long, short) tiles of batch element bb (0 if inconsistent)
    const int n = valid(bb) ? n_chunks[bb] : 0;
    const int32_t* ob = off + (long long)bb * (Nmax + 1);
    int2 local = make_int2(0, 0);
    for (int c = t; c < n; c += 1024) {
      const int2 k = tile_counts(ob[c + 1] - ob[c], policy);
      local.x += k.x;
      local.y += k.y;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      local.x += __shfl_xor_sync(0xffffffffu, local.x, o);
      local.y += __shfl_xor_sync(0xffffffffu, local.y, o);
    }
    __syncthreads();
    if (lane == 0) warp_sum[wp] = local;
    __syncthreads();
    int2 tot = make_int2(0, 0);
    for (int q = 0; q < 32; ++q) {
      tot.x += warp_sum[q].x;
      tot.y += warp_sum[q].y;
    }
    return tot;
  };
  long long base_l = 0, base_s = 0;
  for (int bb = 0; bb < b; ++bb) {
    const int2 tb = totals_of(bb);
    base_l += (long long)Hq * tb.x;
    base_s += (long long)Hq * tb.y;
  }
  const int2 Tb = totals_of(b);
  const bool ok_b = valid(b);
  if (!ok_b && hq == 0 && t == 0) raise_device_flag(status, DHSA_DEVFLAG_BAD_OFFSETS);
  const int n = ok_b ? n_chunks[b] : 0;
  const int32_t* ob = off + (long long)b * (Nmax + 1);
  __syncthreads();
  if (t == 0) carry_s = make_int2(0, 0);
  __syncthreads();
  for (int c0 = 0; c0 < n; c0 += 1024) {
    const int c = c0 + t;
    const int2 k = (c < n) ? tile_counts(ob[c + 1] - ob[c], policy) : make_int2(0, 0);
    int2 incl = k;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int vx = __shfl_up_sync(0xffffffffu, incl.x, o), vy = __shfl_up_sync(0xffffffffu, incl.y, o);
      if (lane >= o) {
        incl.x += vx;
        incl.y += vy;
      }
    }
    if (lane == 31) warp_sum[wp] = incl;
    __syncthreads();
    int2 before = carry_s;
    for (int q = 0; q < wp; ++q) {
      before.x += warp_sum[q].x;
      before.y += warp_sum[q].y;
    }
    const int offl = before.x + incl.x - k.x, offs = before.y + incl.y - k.y;
    for (int tt = 0; tt < k.x; ++tt) {
      const long long idx = base_l + (long long)hkv * G * Tb.x + (long long)G * offl + (long long)gq * k.x + tt;
      w.items_long[idx] = make_int4(b, hq, c, tt);
    }
    for (int tt = 0; tt < k.y; ++tt) {
      const long long idx = base_s + (long long)hkv * G * Tb.y + (long long)G * offs + (long long)gq * k.y + tt;
      w.items_short[idx] = make_int4(b, hq, c, kQueryTileRows * k.x + kShortRows * tt);
    }
    __syncthreads();
    if (t == 1023) carry_s = make_int2(before.x + incl.x, before.y + incl.y);
    __syncthreads();
  }
  if (hq == 0 && b == B - 1 && t == 0) {
    *w.n_long = (int)(base_l + (long long)Hq * Tb.x);
    *w.n_short = (int)(base_s + (long long)Hq * Tb.y);
  }
  if (hq == 0 && b == 0 && t == 0) {   // the attention kernels' item dispensers
    *w.counter_long = 0;
    *w.counter_short = 0;
  }
}

}  // namespace

// Capacities of the two lists for a problem of B x Hq rows of at most Nmax
// chunks over L tokens (a chunk of n tokens has ceil(n / 128) 128-row tiles,
// at most one short tail tile, or ceil(n / 64) 64-row tiles).
long long attn_cap_long(int B, int Hq, int L, int Nmax, int policy) {
  if (policy == 2) return 0;
  return (long long)B * Hq * ((long long)Nmax + ceil_div(L, kQueryTileRows));
}
long long attn_cap_short(int B, int Hq, int L, int Nmax, int policy) {
  if (policy == 0) return 0;
  if (policy == 1) return (long long)B * Hq * Nmax;
  return (long long)B * Hq * ((long long)Nmax + ceil_div(L, kShortRows));
}

int launch_build_items(const int32_t* off, const int32_t* n_chunks, int B, int Hq, int G, int L, int Nmax,
                       int policy, const AttnWork& w, unsigned int* status, cudaStream_t stream) {
  build_items_kernel<<<dim3(Hq, B), 1024, 0, stream>>>(off, n_chunks, B, Hq, G, L, Nmax, policy, w, status);
  return launch_status();
}

}  // namespace dhsa

// Causal block-sparse attention forward over the kept chunk pairs (DHSA stage 5).
//
// DHSA README, "Overview": block-sparse attention extended to variable-sized
// query and key blocks; "Installation": the kernel is BF16, causal,
// forward-only, head dim 128. gist.science technical summary, "Key Technical
// Components": a tiled online-softmax backend that never builds the full
// attention matrix. For query token t of chunk i the kept keys are the tokens
// of the selected chunks (ascending, diagonal chunk last) with s <= t.
//
// sm_100a design
// --------------
// * Work item = (b, hq, query chunk i, 128-row query tile of that chunk).
//   A persistent grid (one CTA per SM) walks a work list in a static
//   round-robin; all roles of a CTA walk the same list.
// * Key stream: the kept chunks of row (b, hq, i) are concatenated and packed
//   into 128-slot key tiles. Each chunk starts on an 8-slot boundary (one
//   128-byte-swizzle atom = 8 rows x 128 B, so every TMA destination is
//   1024-byte aligned) and is fetched with TMA boxes of 64/32/16/8 rows at
//   arbitrary row coordinates. Padding slots and causally hidden keys are
//   masked in registers through a per-tile slot -> token table.
// * Warp roles (192 threads): warp 0 = TMA producer (Q tile, K/V ring of
//   2 stages), warp 1 = tcgen05 MMA issuer (one thread), warps 2-5 = softmax
//   and epilogue (thread = query row = TMEM lane).
// * TMEM (512 columns): S double buffer (2 x 128 fp32 columns) and the O
//   accumulator (128 columns). P = softmax numerators is written back as bf16
//   into the S buffer it came from and consumed from TMEM by the PV MMA
//   (A operand in TMEM, V as an N-major shared-memory operand).
// * Online softmax in the log2 domain; the running max is only raised (and O
//   rescaled in TMEM) when it grows by more than 8 (a factor 256), which keeps
//   the final O / l exact while skipping most rescales.
// * Every mbarrier wait is bounded; a timeout sets DHSA_DEVFLAG_WAIT_TIMEOUT,
//   the CTA drains its own in-flight copies and MMAs (again bounded), frees
//   its TMEM and exits.
#include <cuda.h>

#include "common.cuh"
#include "sm100_ptx.cuh"

namespace dhsa {
namespace {

using namespace ptx;

constexpr int BM = 128;              // query rows per tile
constexpr int BN = 128;              // key slots per tile
constexpr int NS = 2;                // K/V pipeline stages
constexpr int kThreads = 192;
constexpr uint32_t kHalfBytes = 128 * 128;   // 128 rows x 64 bf16 (one 128B-swizzled half tile)
constexpr uint32_t kTileBytes = 2 * kHalfBytes;
constexpr uint32_t kTmemCols = 512;
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s per wait
constexpr int kNoToken = 0x7fffffff;

struct AttnMaps {
  CUtensorMap q;      // box 64 x 128 rows
  CUtensorMap k[4];   // boxes 64 x {8,16,32,64} rows
  CUtensorMap v[4];
};

struct AttnParams {
  const int32_t* off;
  const int32_t* row_ptr;
  const int32_t* col_idx;
  const int4* items;      // (b, hq, i, tile)
  const int* n_items;
  __nv_bfloat16* O;
  int Hq, Hkv, G, L, Nmax;
  float scale_log2;
  unsigned int* status;
};

struct ItemMeta {
  int q0;       // first query token of the tile
  int q_rows;   // valid query rows (1..128)
  int T;        // key tiles
  int pad;
  long long o_row0;  // global row (in O) of token 0 of this (b, hq)
};

// shared-memory layout (offsets from a 1024-aligned base)
constexpr uint32_t OFF_Q = 0;                                   // 2 x 32 KB
constexpr uint32_t OFF_K = OFF_Q + 2 * kTileBytes;              // NS x 32 KB
constexpr uint32_t OFF_V = OFF_K + NS * kTileBytes;             // NS x 32 KB
constexpr uint32_t OFF_TOK = OFF_V + NS * kTileBytes;           // NS x 128 int
constexpr uint32_t OFF_FLAG = OFF_TOK + NS * BN * 4;            // NS int
constexpr uint32_t OFF_META = OFF_FLAG + 16;                    // 2 x ItemMeta
constexpr uint32_t OFF_BAR = OFF_META + 2 * sizeof(ItemMeta);   // barriers (8 B each)
enum {
  B_QFULL = 0, B_QEMPTY = 2, B_IFULL = 4, B_IEMPTY = 6, B_KFULL = 8, B_VFULL = 8 + NS, B_KVEMPTY = 8 + 2 * NS,
  B_SFULL = 8 + 3 * NS, B_PREADY = 10 + 3 * NS, B_ODONE = 12 + 3 * NS, B_FINAL = 13 + 3 * NS, B_COUNT = 14 + 3 * NS
};
constexpr uint32_t OFF_TMEMPTR = OFF_BAR + 8 * B_COUNT;
constexpr uint32_t OFF_ABORT = OFF_TMEMPTR + 4;
constexpr uint32_t kSmemBytes = OFF_ABORT + 4;
constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;  // slack for aligning the base

__device__ __forceinline__ int round8(int x) { return (x + 7) & ~7; }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

struct Flags {
  volatile int* abort;
  unsigned int* status;
  __device__ bool wait(uint32_t bar, uint32_t parity) {
    if (*abort) return false;
    if (mbar_wait(bar, parity, kWaitLimitNs)) return true;
    *abort = 1;
    raise_device_flag(status, DHSA_DEVFLAG_WAIT_TIMEOUT);
    return false;
  }
};

__global__ void __launch_bounds__(kThreads, 1) sparse_attn_fwd_kernel(const __grid_constant__ AttnMaps maps,
                                                                      const AttnParams p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  int* slot_tok = reinterpret_cast<int*>(smem + OFF_TOK);
  int* tile_flag = reinterpret_cast<int*>(smem + OFF_FLAG);
  ItemMeta* meta = reinterpret_cast<ItemMeta*>(smem + OFF_META);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_ABORT);
  auto bar = [&](int idx) { return sbase + OFF_BAR + 8u * idx; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_items = *p.n_items;

  // ---------------------------------------------------------------- setup
  if (warp == 0) {
    if (lane == 0) {
      *abort_flag = 0;
      for (int s = 0; s < 2; ++s) {
        mbar_init(bar(B_QFULL + s), 1);
        mbar_init(bar(B_QEMPTY + s), 1);
        mbar_init(bar(B_IFULL + s), 1);
        mbar_init(bar(B_IEMPTY + s), 5);   // MMA thread + 4 softmax warps
        mbar_init(bar(B_SFULL + s), 1);
        mbar_init(bar(B_PREADY + s), 4);   // 4 softmax warps
      }
      for (int s = 0; s < NS; ++s) {
        mbar_init(bar(B_KFULL + s), 1);
        mbar_init(bar(B_VFULL + s), 1);
        mbar_init(bar(B_KVEMPTY + s), 1);
      }
      mbar_init(bar(B_ODONE), 1);
      mbar_init(bar(B_FINAL), 1);
      fence_mbar_init();
      prefetch_tmap(&maps.q);
      for (int s = 0; s < 4; ++s) {
        prefetch_tmap(&maps.k[s]);
        prefetch_tmap(&maps.v[s]);
      }
    }
  } else if (warp == 1) {
    tmem_alloc(sbase + OFF_TMEMPTR, kTmemCols);
    tmem_relinquish();
  }
  // V slots that no TMA ever fills must hold finite values (a masked key
  // contributes P = 0 times its V row); zero both V stages once.
  for (uint32_t o = threadIdx.x * 16; o < NS * kTileBytes; o += kThreads * 16)
    *reinterpret_cast<uint4*>(smem + OFF_V + o) = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + OFF_TMEMPTR);
  Flags fl{abort_flag, p.status};

  if (warp == 0) {
    // ============================================================ producer
    uint32_t g = 0;  // global key-tile counter of this CTA
    int n_local = 0;
    for (int it = blockIdx.x; it < n_items && !*abort_flag; it += gridDim.x, ++n_local) {
      const int4 wi = p.items[it];
      const int b = wi.x, hq = wi.y, i = wi.z, tq = wi.w;
      const int32_t* ob = p.off + (long long)b * (p.Nmax + 1);
      const int c_start = ob[i], c_end = ob[i + 1];
      const int q0 = c_start + BM * tq;
      const int q_rows = min(BM, c_end - q0);
      const int q_last = q0 + q_rows - 1;
      const long long r = ((long long)b * p.Hq + hq) * p.Nmax + i;
      const int rp0 = p.row_ptr[r], rp1 = p.row_ptr[r + 1];
      const long long kv_row0 = ((long long)b * p.Hkv + hq / p.G) * p.L;
      const long long q_row0 = ((long long)b * p.Hq + hq) * p.L;

      // first batch of chunk descriptors in lanes, and the total slot count
      int cj = -1, cst = 0, clen = 0, slots = 0;
      for (int q = rp0 + lane; q < rp1; q += 32) {
        const int j = p.col_idx[q];
        const int s0 = ob[j];
        const int len = (j == i) ? (q_last + 1 - c_start) : (ob[j + 1] - s0);
        slots += round8(len);
        if (q < rp0 + 32) { cj = j; cst = s0; clen = len; }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) slots += __shfl_xor_sync(0xffffffffu, slots, o);
      const int T = (slots + BN - 1) / BN;

      const int ms = n_local & 1;
      if (n_local >= 2 && !fl.wait(bar(B_IEMPTY + ms), ((n_local >> 1) - 1) & 1)) break;
      if (lane == 0) {
        meta[ms].q0 = q0;
        meta[ms].q_rows = q_rows;
        meta[ms].T = T;
        meta[ms].o_row0 = q_row0;
        mbar_arrive(bar(B_IFULL + ms));
      }
      if (n_local >= 2 && !fl.wait(bar(B_QEMPTY + ms), ((n_local >> 1) - 1) & 1)) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(bar(B_QFULL + ms), kTileBytes);
        const uint32_t dq = sbase + OFF_Q + ms * kTileBytes;
        tma_load_2d(dq, &maps.q, bar(B_QFULL + ms), 0, (int)(q_row0 + q0));
        tma_load_2d(dq + kHalfBytes, &maps.q, bar(B_QFULL + ms), 64, (int)(q_row0 + q0));
      }

      int seg_q = rp0, cur = 0, seg_pos = 0;
      bool ok = true;
      for (int kt = 0; kt < T; ++kt, ++g) {
        const int st = g % NS;
        if (g >= NS && !fl.wait(bar(B_KVEMPTY + st), ((g / NS) - 1) & 1)) { ok = false; break; }
        int slot = 0, needs_mask = 0;
        int* tok = slot_tok + st * BN;
        const uint32_t dk = sbase + OFF_K + st * kTileBytes;
        const uint32_t dv = sbase + OFF_V + st * kTileBytes;
        while (slot < BN && seg_q < rp1) {
          const int j = __shfl_sync(0xffffffffu, cj, cur);
          const int s0 = __shfl_sync(0xffffffffu, cst, cur);
          const int len = __shfl_sync(0xffffffffu, clen, cur);
          const int rows = min(len - seg_pos, BN - slot);
          const int groups = (rows + 7) >> 3;
          const int tok0 = s0 + seg_pos;
          for (int s = lane; s < groups * 8; s += 32) tok[slot + s] = (s < rows) ? tok0 + s : kNoToken;
          if (rows < groups * 8 || j == i) needs_mask = 1;
          if (lane == 0) {
            int gq = 0;
            while (gq < groups) {
              const int rem = groups - gq;
              const int bx = rem >= 8 ? 3 : rem >= 4 ? 2 : rem >= 2 ? 1 : 0;
              const int nrows = 8 << bx;
              const uint32_t bytes = nrows * 128u;
              const int y = (int)(kv_row0 + tok0 + 8 * gq);
              const uint32_t so = (uint32_t)(slot + 8 * gq) * 128u;
              mbar_expect_tx(bar(B_KFULL + st), 2 * bytes);
              tma_load_2d(dk + so, &maps.k[bx], bar(B_KFULL + st), 0, y);
              tma_load_2d(dk + kHalfBytes + so, &maps.k[bx], bar(B_KFULL + st), 64, y);
              mbar_expect_tx(bar(B_VFULL + st), 2 * bytes);
              tma_load_2d(dv + so, &maps.v[bx], bar(B_VFULL + st), 0, y);
              tma_load_2d(dv + kHalfBytes + so, &maps.v[bx], bar(B_VFULL + st), 64, y);
              gq += nrows >> 3;
            }
          }
          slot += groups * 8;
          seg_pos += rows;
          if (seg_pos == len) {
            seg_pos = 0;
            ++seg_q;
            if (++cur == 32 && seg_q < rp1) {
              cur = 0;
              const int q = seg_q + lane;
              if (q < rp1) {
                const int jj = p.col_idx[q];
                cj = jj;
                cst = ob[jj];
                clen = (jj == i) ? (q_last + 1 - c_start) : (ob[jj + 1] - cst);
              }
            }
          }
        }
        for (int s = slot + lane; s < BN; s += 32) tok[s] = kNoToken;
        if (slot < BN) needs_mask = 1;
        if (lane == 0) tile_flag[st] = needs_mask;
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(bar(B_KFULL + st));
          mbar_arrive(bar(B_VFULL + st));
        }
      }
      if (!ok) break;
    }
    // drain: every copy this warp issued must have landed before teardown
    if (lane == 0) {
      for (uint32_t gg = (g > NS ? g - NS : 0); gg < g; ++gg) {
        const int st = gg % NS;
        mbar_wait(bar(B_KFULL + st), (gg / NS) & 1, kWaitLimitNs);
        mbar_wait(bar(B_VFULL + st), (gg / NS) & 1, kWaitLimitNs);
      }
      for (int n = (n_local > 2 ? n_local - 2 : 0); n < n_local; ++n)
        mbar_wait(bar(B_QFULL + (n & 1)), (n >> 1) & 1, kWaitLimitNs);
    }
  } else if (warp == 1) {
    // ============================================================ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_qk = idesc_bf16_f32(BM, BN, false);
      const uint32_t idesc_pv = idesc_bf16_f32(BM, 128, true);
      const uint32_t tS0 = tmem, tO = tmem + 256;
      uint32_t g = 0;
      int n_local = 0;
      auto issue_pv = [&](uint32_t u, bool first) -> bool {
        const int st = u % NS, sb = u & 1;
        if (!fl.wait(bar(B_PREADY + sb), (u >> 1) & 1)) return false;
        if (!fl.wait(bar(B_VFULL + st), (u / NS) & 1)) return false;
        tc_fence_after();
        const uint32_t v0 = sbase + OFF_V + st * kTileBytes;
#pragma unroll
        for (int ks = 0; ks < BN / 16; ++ks) {
          const uint64_t bdesc = smem_desc_sw128(v0 + ks * 2048, kHalfBytes, 1024);
          mma_ts(tO, tS0 + sb * 128 + ks * 8, bdesc, idesc_pv, (!first || ks > 0) ? 1u : 0u);
        }
        mma_commit(bar(B_KVEMPTY + st));
        mma_commit(bar(B_ODONE));
        return true;
      };
      for (int it = blockIdx.x; it < n_items; it += gridDim.x, ++n_local) {
        const int ms = n_local & 1;
        if (!fl.wait(bar(B_IFULL + ms), (n_local >> 1) & 1)) break;
        const int T = meta[ms].T;
        mbar_arrive(bar(B_IEMPTY + ms));
        if (!fl.wait(bar(B_QFULL + ms), (n_local >> 1) & 1)) break;
        const uint32_t q0 = sbase + OFF_Q + ms * kTileBytes;
        bool ok = true;
        for (int kt = 0; kt < T; ++kt, ++g) {
          const int st = g % NS, sb = g & 1;
          if (!fl.wait(bar(B_KFULL + st), (g / NS) & 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t k0 = sbase + OFF_K + st * kTileBytes;
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const uint32_t ko = (ks >> 2) * kHalfBytes + (ks & 3) * 32;
            const uint64_t adesc = smem_desc_sw128(q0 + ko, 16, 1024);
            const uint64_t bdesc = smem_desc_sw128(k0 + ko, 16, 1024);
            mma_ss(tS0 + sb * 128, adesc, bdesc, idesc_qk, ks > 0 ? 1u : 0u);
          }
          mma_commit(bar(B_SFULL + sb));
          if (kt == T - 1) mma_commit(bar(B_QEMPTY + ms));
          if (kt >= 1 && !issue_pv(g - 1, kt == 1)) { ok = false; break; }
        }
        if (!ok) break;
        if (T == 0) {
          mma_commit(bar(B_QEMPTY + ms));   // an empty key set: nothing to multiply
        } else if (!issue_pv(g - 1, T == 1)) {
          break;
        }
      }
      // drain the tensor pipe before TMEM is released
      mma_commit(bar(B_FINAL));
      mbar_wait(bar(B_FINAL), 0, kWaitLimitNs);
    }
  } else {
    // ============================================================ softmax + epilogue
    const int quarter = warp & 3;             // TMEM lanes 32*quarter .. +31
    const int row = quarter * 32 + lane;      // query row within the tile
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS0 = tmem + lane_addr, tO = tmem + lane_addr + 256;
    uint32_t g = 0, pv_seen = 0;
    int n_local = 0;
    for (int it = blockIdx.x; it < n_items; it += gridDim.x, ++n_local) {
      const int ms = n_local & 1;
      if (!fl.wait(bar(B_IFULL + ms), (n_local >> 1) & 1)) break;
      const ItemMeta mt = meta[ms];
      const int qt = mt.q0 + row;
      float m_used = -INFINITY, l_sum = 0.f;
      bool ok = true;
      for (int kt = 0; kt < mt.T; ++kt, ++g) {
        const int st = g % NS, sb = g & 1;
        if (!fl.wait(bar(B_SFULL + sb), (g >> 1) & 1) || !fl.wait(bar(B_KFULL + st), (g / NS) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t s[BN];
        tmem_ld32(tS0 + sb * 128 + 0, *reinterpret_cast<uint32_t(*)[32]>(s + 0));
        tmem_ld32(tS0 + sb * 128 + 32, *reinterpret_cast<uint32_t(*)[32]>(s + 32));
        tmem_ld32(tS0 + sb * 128 + 64, *reinterpret_cast<uint32_t(*)[32]>(s + 64));
        tmem_ld32(tS0 + sb * 128 + 96, *reinterpret_cast<uint32_t(*)[32]>(s + 96));
        tmem_wait_ld();
        float mx = -INFINITY;
        if (tile_flag[st]) {
          const int4* tok4 = reinterpret_cast<const int4*>(slot_tok + st * BN);
#pragma unroll
          for (int c4 = 0; c4 < BN / 4; ++c4) {
            const int4 tk = tok4[c4];
            const int tks[4] = {tk.x, tk.y, tk.z, tk.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int c = 4 * c4 + e;
              const float v = (tks[e] <= qt) ? __uint_as_float(s[c]) * p.scale_log2 : -INFINITY;
              s[c] = __float_as_uint(v);
              mx = fmaxf(mx, v);
            }
          }
        } else {
#pragma unroll
          for (int c = 0; c < BN; ++c) {
            const float v = __uint_as_float(s[c]) * p.scale_log2;
            s[c] = __float_as_uint(v);
            mx = fmaxf(mx, v);
          }
        }
        const float m_new = fmaxf(m_used, mx);
        const bool rescale = m_new > m_used + 8.0f;  // also true on the first tile
        if (kt > 0) {
          // PV of the previous tile must be complete before O is touched or
          // its P buffer's neighbour is overwritten
          if (!fl.wait(bar(B_ODONE), pv_seen & 1)) { ok = false; break; }
          ++pv_seen;
          tc_fence_after();
          if (__any_sync(0xffffffffu, rescale)) {
            const float f = rescale ? fast_exp2(m_used - m_new) : 1.f;
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
              uint32_t o[32];
              tmem_ld32(tO + 32 * c4, o);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
              tmem_st32(tO + 32 * c4, o);
            }
            tmem_wait_st();
            if (rescale) l_sum *= f;
          }
        }
        if (rescale) m_used = m_new;
        float rs = 0.f;
        uint32_t pk[BN / 2];
#pragma unroll
        for (int c = 0; c < BN / 2; ++c) {
          const float p0 = fast_exp2(__uint_as_float(s[2 * c]) - m_used);
          const float p1 = fast_exp2(__uint_as_float(s[2 * c + 1]) - m_used);
          rs += p0 + p1;
          pk[c] = pack_bf16x2(p0, p1);
        }
        l_sum += rs;
        tmem_st32(tS0 + sb * 128 + 0, *reinterpret_cast<uint32_t(*)[32]>(pk + 0));
        tmem_st32(tS0 + sb * 128 + 32, *reinterpret_cast<uint32_t(*)[32]>(pk + 32));
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_PREADY + sb));
      }
      if (!ok) break;
      // epilogue: O / l -> bf16 (an empty key set, which valid CSR input never
      // has, writes zeros)
      if (mt.T > 0) {
        if (!fl.wait(bar(B_ODONE), pv_seen & 1)) break;
        ++pv_seen;
      }
      tc_fence_after();
      const float inv_l = mt.T > 0 ? 1.f / l_sum : 0.f;
      __nv_bfloat16* orow = p.O + (mt.o_row0 + qt) * kHeadDim;
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        uint32_t o[32];
        tmem_ld32(tO + 32 * c4, o);
        tmem_wait_ld();
        if (mt.T == 0) {
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = 0u;
        }
        if (row < mt.q_rows) {
          uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c4);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(o[8 * v + 0]) * inv_l, __uint_as_float(o[8 * v + 1]) * inv_l);
            w.y = pack_bf16x2(__uint_as_float(o[8 * v + 2]) * inv_l, __uint_as_float(o[8 * v + 3]) * inv_l);
            w.z = pack_bf16x2(__uint_as_float(o[8 * v + 4]) * inv_l, __uint_as_float(o[8 * v + 5]) * inv_l);
            w.w = pack_bf16x2(__uint_as_float(o[8 * v + 6]) * inv_l, __uint_as_float(o[8 * v + 7]) * inv_l);
            dst[v] = w;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_IEMPTY + ms));
    }
  }

  // ---------------------------------------------------------------- teardown
  __syncwarp();  // lanes that waited out their role's single-thread work reconverge here
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

// Work list: one item per (b, hq, chunk i, 128-row tile of i), ordered
// (b, kv head, i, query head within the group, tile) so that CTAs running at
// the same time share the K/V of one kv head in L2.
__global__ void __launch_bounds__(1024) build_items_kernel(const int32_t* __restrict__ off,
                                                           const int32_t* __restrict__ n_chunks, int B, int Hq,
                                                           int G, int Nmax, int4* __restrict__ items,
                                                           int* __restrict__ n_items) {
  __shared__ int warp_sum[32];
  __shared__ int carry_s;
  const int t = threadIdx.x, lane = t & 31, w = t >> 5;
  const int Hkv = Hq / G;
  long long base = 0;
  for (int b = 0; b < B; ++b) {
    const int n = n_chunks[b];
    const int32_t* ob = off + (long long)b * (Nmax + 1);
    // pass 1: tiles of this batch element
    int local = 0;
    for (int c = t; c < n; c += 1024) local += (ob[c + 1] - ob[c] + BM - 1) / BM;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) local += __shfl_xor_sync(0xffffffffu, local, o);
    if (lane == 0) warp_sum[w] = local;
    __syncthreads();
    int Tb = 0;
    for (int q = 0; q < 32; ++q) Tb += warp_sum[q];
    __syncthreads();
    // pass 2: running exclusive scan of tiles per chunk, then write items
    if (t == 0) carry_s = 0;
    __syncthreads();
    for (int c0 = 0; c0 < n; c0 += 1024) {
      const int c = c0 + t;
      const int tiles = (c < n) ? (ob[c + 1] - ob[c] + BM - 1) / BM : 0;
      int incl = tiles;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      if (lane == 31) warp_sum[w] = incl;
      __syncthreads();
      int before = carry_s;
      for (int q = 0; q < w; ++q) before += warp_sum[q];
      const int toff = before + incl - tiles;
      for (int hkv = 0; hkv < Hkv; ++hkv)
        for (int gq = 0; gq < G; ++gq)
          for (int tt = 0; tt < tiles; ++tt) {
            const long long idx = base + (long long)hkv * G * Tb + (long long)G * toff + (long long)gq * tiles + tt;
            items[idx] = make_int4(b, hkv * G + gq, c, tt);
          }
      __syncthreads();
      if (t == 1023) carry_s = before + incl;
      __syncthreads();
    }
    base += (long long)Hq * Tb;
  }
  if (t == 0) *n_items = (int)base;
}

// --------------------------------------------------------------------- host
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

bool make_map(EncodeTiledFn enc, CUtensorMap* m, const void* base, long long rows, int box_rows) {
  const cuuint64_t dims[2] = {(cuuint64_t)kHeadDim, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)kHeadDim * 2};
  const cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1u, 1u};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// ----------------------------------------------------------- no-allocation variant
// Scratch for callers that must not allocate device memory. It lives in a
// file-scope device array that every GPU loading the library holds until the
// process exits. It backs the same work list the caller's workspace would
// hold, so the maximum problem is the one whose work list fits:
// 256 + 16 * B * Hq * (Nmax + ceil(L / 128)) bytes <= 4 MiB.
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
constexpr int kNoAllocMaxDevices = 64;
void* g_noalloc_ptr[kNoAllocMaxDevices] = {nullptr};
}  // namespace

size_t attn_items_cap(int B, int Hq, int L, int Nmax) {
  return (size_t)B * Hq * ((size_t)Nmax + (size_t)(L + BM - 1) / BM);
}

size_t attn_ws_bytes(int B, int Hq, int L, int Nmax) { return 256 + sizeof(int4) * attn_items_cap(B, Hq, L, Nmax); }

int launch_sparse_attn(const void* Q, const void* K, const void* V, int B, int Hq, int Hkv, int L,
                       const int32_t* off, const int32_t* n_chunks, int Nmax, const int32_t* row_ptr,
                       const int32_t* col_idx, float softmax_scale, void* O, void* ws, unsigned int* status,
                       cudaStream_t stream) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return cuda_status(cudaErrorNotSupported);
  AttnMaps maps;
  const long long q_rows = (long long)B * Hq * L, kv_rows = (long long)B * Hkv * L;
  bool ok = make_map(enc, &maps.q, Q, q_rows, BM);
  for (int s = 0; s < 4; ++s) {
    ok = ok && make_map(enc, &maps.k[s], K, kv_rows, 8 << s);
    ok = ok && make_map(enc, &maps.v[s], V, kv_rows, 8 << s);
  }
  if (!ok) return DHSA_ERR_INVALID_ARG;

  int* n_items = static_cast<int*>(ws);
  int4* items = reinterpret_cast<int4*>(static_cast<char*>(ws) + 256);
  build_items_kernel<<<1, 1024, 0, stream>>>(off, n_chunks, B, Hq, Hq / Hkv, Nmax, items, n_items);
  int st = launch_status();
  if (st != DHSA_OK) return st;

  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(sparse_attn_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemAlloc);
  if (e != cudaSuccess) return cuda_status(e);

  AttnParams prm;
  prm.off = off;
  prm.row_ptr = row_ptr;
  prm.col_idx = col_idx;
  prm.items = items;
  prm.n_items = n_items;
  prm.O = static_cast<__nv_bfloat16*>(O);
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.G = Hq / Hkv;
  prm.L = L;
  prm.Nmax = Nmax;
  prm.scale_log2 = softmax_scale * 1.4426950408889634f;
  prm.status = status;
  const long long cap = (long long)attn_items_cap(B, Hq, L, Nmax);
  const int grid = (int)(cap < sms ? cap : sms);
  sparse_attn_fwd_kernel<<<grid, kThreads, kSmemAlloc, stream>>>(maps, prm);
  return launch_status();
}

}  // namespace dhsa

namespace dhsa {

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

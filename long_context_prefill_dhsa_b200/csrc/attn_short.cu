// Causal block-sparse attention forward for short query tiles (at most 64
// query rows of one chunk): the computation of attn_fwd.cu (DHSA README,
// "Overview" and "Installation"; gist.science technical summary, "Key
// Technical Components": a tiled online softmax over the kept keys), arranged
// for the tail tiles of chunks, whose rows would leave most of a 128-row
// query tile empty.
//
// sm_100a design
// --------------
// * Transposed tiles: the 128 key slots of a key tile are the MMA's M
//   dimension and the item's (up to 64) query rows its N dimension, so each
//   MMA instruction costs about N/2 = 32 tensor cycles (an M = 64 tile would
//   cost as much as M = 128). S^T = K Q^T takes both operands K-major from
//   their 128-byte-swizzled TMA tiles and lands in TMEM with one key slot per
//   lane. O^T += V^T P^T reads V^T straight from the V tile and P^T from
//   shared memory, both as M/N-major (128-byte swizzle) operands.
// * Softmax in the log2 domain, per query column over the key slots. A thread
//   owns one key slot (a TMEM lane); warpgroup 1 takes query columns 0..31
//   and warpgroup 2 columns 32..63, so the two never exchange anything. The
//   running max of each column is kept (as its negation) in shared memory and
//   is only raised when a score exceeds it by more than 2^32; the four warps
//   of a warpgroup agree on that with one barrier reduction per tile. A raise
//   (and the first tile of every item) takes the column maxima over the 128
//   slots (warp max reductions, then shared memory), rescales this thread's
//   partial row sums and its row of O^T in TMEM, and publishes the new max.
//   Row sums stay per thread until the epilogue reduces them.
// * Masking: a 128-bit valid-slot mask per tile (padding slots give p = 0)
//   and, in the diagonal chunk's piece, per slot the first query column that
//   may see it.
// * Warp roles (512 threads): warp 0 = TMA producer of Q and K, warp 3 = TMA
//   producer of V, warp 1 = S^T issuer, warp 14 = O^T issuer (one thread
//   each), warp 2 = scheduler (takes the next short item from its work list
//   by atomic counter), warps 4-11 = softmax + epilogue.
// * TMEM (256 columns): three S^T buffers of 64 columns, O^T (64 columns).
//   Shared memory: Q (2 x 16 KB), K and V rings (2 x 32 KB each), three P^T
//   buffers (16 KB each).
// * Every mbarrier wait is bounded; a timeout sets DHSA_DEVFLAG_WAIT_TIMEOUT
//   and the CTA drains and exits. The warpgroup barriers are only ever
//   reached by all four warps of the group: every exit decision is taken from
//   a barrier reduction, so the four warps leave together.
#include <cuda.h>

#include "common.cuh"
#include "sm100_ptx.cuh"
#include "tmap.cuh"

namespace dhsa {
namespace {

using namespace ptx;

constexpr int BN = 128;              // key slots per tile (MMA M)
constexpr int NQ = 64;               // query rows per short tile (MMA N)
constexpr int NSK = 2, NSV = 2;      // K and V pipeline stages
constexpr int NSB = 3;               // S^T buffers in TMEM, P^T buffers in shared memory
constexpr int NTOK = 4;              // tile descriptor ring
constexpr int NSLOT = 4;             // scheduled work items in flight
constexpr int SEG_CAP = 64;          // chunk descriptors kept in shared memory per item
constexpr int kThreads = 512;
constexpr uint32_t kKHalf = 128 * 128;          // 128 key rows x 64 bf16
constexpr uint32_t kKTile = 2 * kKHalf;
constexpr uint32_t kQHalf = NQ * 128;           // 64 query rows x 64 bf16
constexpr uint32_t kQTile = 2 * kQHalf;
constexpr uint32_t kPTile = BN * NQ * 2;        // P^T: 128 key rows x 64 bf16
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kTmemO = 192;                // O^T columns
constexpr float kRaise = 32.0f;                 // log2 headroom before a column max must rise

struct ShortMaps {
  CUtensorMap q;      // box 64 cols x 64 rows
  CUtensorMap k[16];  // boxes 64 cols x 8*(n+1) rows
  CUtensorMap v[16];
};

struct ShortParams {
  const int32_t* off;
  const int32_t* row_ptr;
  const int32_t* col_idx;
  const int4* items;      // (b, hq, i, first row of the tile within chunk i)
  const int* n_items;
  int* work_counter;
  __nv_bfloat16* O;
  int Hq, Hkv, G, L, Nmax;
  float scale_log2;
  unsigned int* status;
};

struct ItemMeta {
  int q0;        // token of the first query row
  int q_rows;    // valid query rows (1..64)
  int T;         // key tiles (-1: end of the work list)
  int nseg;      // kept chunks (the last one is the diagonal chunk)
  int kv_row0;   // global K/V row of token 0 of this (b, kv head)
  int q_row0;    // global Q/O row of token 0 of this (b, q head)
  int rp0;       // first CSR entry of the row
  int b;
  int i;         // query chunk
  int c_start;   // first token of chunk i
  int pad[2];
};
struct ItemSlot {
  ItemMeta m;
  int2 seg[SEG_CAP];   // (first token, visible length) of the first SEG_CAP kept chunks
};
// per key tile: valid-slot mask; causal piece: slots s >= d_slot hold token s - d_off
struct TileInfo {
  uint32_t mask[4];
  int causal, d_slot, d_off, pad;
};

// shared-memory layout (offsets from a 1024-aligned base)
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_K = OFF_Q + 2 * kQTile;
constexpr uint32_t OFF_V = OFF_K + NSK * kKTile;
constexpr uint32_t OFF_P = OFF_V + NSV * kKTile;
constexpr uint32_t OFF_TINFO = OFF_P + NSB * kPTile;
constexpr uint32_t OFF_SLOT = OFF_TINFO + NTOK * sizeof(TileInfo);
constexpr uint32_t OFF_NM = OFF_SLOT + NSLOT * sizeof(ItemSlot);   // [half][buffer][32]: -max per column
constexpr uint32_t OFF_RED = OFF_NM + 2 * 2 * 32 * 4;               // [half][quarter][32]: column max keys
constexpr uint32_t OFF_LRED = OFF_RED + 2 * 4 * 32 * 4;             // [half][quarter][32]: row-sum partials
constexpr uint32_t OFF_BAR = OFF_LRED + 2 * 4 * 32 * 4;
enum {
  B_QFULL = 0,
  B_QEMPTY = B_QFULL + 2,
  B_SLFULL = B_QEMPTY + 2,
  B_SLEMPTY = B_SLFULL + NSLOT,
  B_KFULL = B_SLEMPTY + NSLOT,
  B_VFULL = B_KFULL + NSK,
  B_TOKFULL = B_VFULL + NSV,
  B_TOKEMPTY = B_TOKFULL + NTOK,
  B_SFULL = B_TOKEMPTY + NTOK,    // S^T(g) complete: K stage free
  B_SREAD = B_SFULL + NSB,        // the softmax has read S^T(g): buffer free
  B_PREADY = B_SREAD + NSB,       // P^T(g) written
  B_PVDONE = B_PREADY + NSB,      // O^T += V^T P^T(g) complete: P^T buffer and V stage free
  B_OFINAL = B_PVDONE + NSB,
  B_EPIDONE = B_OFINAL + 1,       // the epilogue has read O^T
  B_FINAL = B_EPIDONE + 1,
  B_FINALPV = B_FINAL + 1,
  B_TEARDOWN = B_FINALPV + 1,
  B_COUNT = B_TEARDOWN + 1
};
constexpr uint32_t OFF_TMEMPTR = OFF_BAR + 8 * B_COUNT;
constexpr uint32_t OFF_ABORT = OFF_TMEMPTR + 4;
constexpr uint32_t kSmemBytes = OFF_ABORT + 4;
constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;
static_assert(kSmemAlloc <= 227 * 1024, "shared memory budget");
static_assert(OFF_BAR % 8 == 0 && OFF_SLOT % 16 == 0 && OFF_TINFO % 16 == 0 && OFF_NM % 16 == 0, "alignment");
static_assert(OFF_K % 1024 == 0 && OFF_V % 1024 == 0 && OFF_P % 1024 == 0 && kQHalf % 1024 == 0,
              "128-byte swizzle atoms");

constexpr int W_KPROD = 0, W_QK = 1, W_SCHED = 2, W_VPROD = 3, W_SOFTMAX0 = 4, W_PV = 14;
constexpr int kSoftmaxWarps = 8;
constexpr int kSlotConsumers = 2 + 2 + kSoftmaxWarps;
constexpr uint32_t kRegsLaunch = 65536 / kThreads / 8 * 8;   // 128
constexpr uint32_t kRegsWg0 = 96, kRegsWg3 = 64, kRegsSoftmax = 176;
static_assert(128 * (kRegsWg0 + kRegsWg3 + 2 * kRegsSoftmax) <= kRegsLaunch * kThreads, "register split");

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

__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// order-preserving map of a float to an unsigned key, for integer max reductions
__device__ __forceinline__ unsigned fkey(float f) {
  const unsigned u = __float_as_uint(f);
  return (u >> 31) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float unfkey(unsigned k) { return __uint_as_float((k >> 31) ? (k & 0x7fffffffu) : ~k); }

__device__ __forceinline__ unsigned warp_max_u32(unsigned v) {
  unsigned r;
  asm volatile("redux.sync.max.u32 %0, %1, 0xffffffff;" : "=r"(r) : "r"(v));
  return r;
}

// Barrier over the 128 threads of one softmax warpgroup (named barrier `id`),
// returning whether any participating thread passed `pred`. Orders the
// group's shared-memory accesses like __syncthreads does for the block.
__device__ __forceinline__ bool group_any(int id, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, %2, 128, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void group_sync(int id) { asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory"); }

// instruction descriptor, kind::f16, bf16 operands, f32 accumulator; a_mn /
// b_mn: A (B) stored M- (N-) contiguous
__device__ __forceinline__ uint32_t idesc_tr(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// bits [a, b) of word w of a 128-bit slot mask
__device__ __forceinline__ uint32_t mask_bits(int a, int b, int w) {
  const int lo = max(a, 32 * w) - 32 * w, hi = min(b, 32 * w + 32) - 32 * w;
  if (hi <= lo) return 0u;
  const uint32_t ones = (hi - lo == 32) ? 0xffffffffu : ((1u << (hi - lo)) - 1u);
  return ones << lo;
}

struct Flags {
  volatile int* abort;
  unsigned int* status;
  __device__ __forceinline__ bool wait(uint32_t bar, uint32_t parity) {
    if (mbar_test_wait(bar, parity)) return true;
    if (*abort) return false;
    if (mbar_wait_slow(bar, parity, kWaitLimitNs)) return true;
    *abort = 1;
    raise_device_flag(status, DHSA_DEVFLAG_WAIT_TIMEOUT);
    return false;
  }
};

__global__ void __launch_bounds__(kThreads, 1) sparse_attn_short_kernel(const __grid_constant__ ShortMaps maps,
                                                                       const ShortParams p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  TileInfo* tile_info = reinterpret_cast<TileInfo*>(smem + OFF_TINFO);
  ItemSlot* slots = reinterpret_cast<ItemSlot*>(smem + OFF_SLOT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_ABORT);
  auto bar = [&](int idx) { return sbase + OFF_BAR + 8u * idx; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_items = *p.n_items;

  // ---------------------------------------------------------------- setup
  if (warp == W_KPROD) {
    if (lane == 0) {
      *abort_flag = 0;
      for (int s = 0; s < 2; ++s) {
        mbar_init(bar(B_QFULL + s), 1);
        mbar_init(bar(B_QEMPTY + s), 1);
      }
      for (int s = 0; s < NSLOT; ++s) {
        mbar_init(bar(B_SLFULL + s), 1);
        mbar_init(bar(B_SLEMPTY + s), kSlotConsumers);
      }
      for (int s = 0; s < NSK; ++s) mbar_init(bar(B_KFULL + s), 1);
      for (int s = 0; s < NSV; ++s) mbar_init(bar(B_VFULL + s), 1);
      for (int s = 0; s < NTOK; ++s) {
        mbar_init(bar(B_TOKFULL + s), 1);
        mbar_init(bar(B_TOKEMPTY + s), kSoftmaxWarps);
      }
      for (int s = 0; s < NSB; ++s) {
        mbar_init(bar(B_SFULL + s), 1);
        mbar_init(bar(B_SREAD + s), kSoftmaxWarps);
        mbar_init(bar(B_PREADY + s), kSoftmaxWarps);
        mbar_init(bar(B_PVDONE + s), 1);
      }
      mbar_init(bar(B_OFINAL), 1);
      mbar_init(bar(B_EPIDONE), kSoftmaxWarps);
      mbar_init(bar(B_FINAL), 1);
      mbar_init(bar(B_FINALPV), 1);
      mbar_init(bar(B_TEARDOWN), kThreads / 32 - 1);
      fence_mbar_init();
      prefetch_tmap(&maps.q);
      for (int s = 0; s < 16; ++s) {
        prefetch_tmap(&maps.k[s]);
        prefetch_tmap(&maps.v[s]);
      }
    }
  } else if (warp == W_QK) {
    tmem_alloc(sbase + OFF_TMEMPTR, kTmemCols);
    tmem_relinquish();
  }
  // Slots that no TMA fills hold finite values (zeros, or keys of an earlier
  // tile): their scores are discarded by the slot mask and their V rows meet
  // p = 0. Zero the K and V rings once.
  for (uint32_t o = threadIdx.x * 16; o < OFF_P - OFF_K; o += kThreads * 16)
    *reinterpret_cast<uint4*>(smem + OFF_K + o) = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + OFF_TMEMPTR);
  Flags fl{abort_flag, p.status};
  if (warp < W_SOFTMAX0) regs_dec<kRegsWg0>();
  else if (warp >= W_SOFTMAX0 + kSoftmaxWarps) regs_dec<kRegsWg3>();

  if (warp == W_SCHED) {
    // ============================================================ scheduler
    int n_local = 0;
    for (;; ++n_local) {
      const int sl = n_local % NSLOT;
      if (n_local >= NSLOT && !fl.wait(bar(B_SLEMPTY + sl), ((n_local / NSLOT) - 1) & 1)) break;
      int it = 0;
      if (lane == 0) it = atomicAdd(p.work_counter, 1);
      it = __shfl_sync(0xffffffffu, it, 0);
      if (it >= n_items) {
        if (lane == 0) {
          slots[sl].m.T = -1;
          mbar_arrive(bar(B_SLFULL + sl));
        }
        break;
      }
      const int4 wi = p.items[it];
      const int b = wi.x, hq = wi.y, i = wi.z;
      const int32_t* ob = p.off + (long long)b * (p.Nmax + 1);
      const int c_start = ob[i], c_end = ob[i + 1];
      const int q0 = c_start + wi.w;
      const int q_rows = min(NQ, c_end - q0);
      const long long r = ((long long)b * p.Hq + hq) * p.Nmax + i;
      const int rp0 = p.row_ptr[r], rp1 = p.row_ptr[r + 1];
      ItemSlot& S = slots[sl];
      int nslots = 0;
      for (int q = rp0 + lane; q < rp1; q += 32) {
        const int j = p.col_idx[q];
        const int s0 = ob[j];
        const int len = (j == i) ? (q0 + q_rows - c_start) : (ob[j + 1] - s0);
        nslots += round8(len);
        if (q - rp0 < SEG_CAP) S.seg[q - rp0] = make_int2(s0, len);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) nslots += __shfl_xor_sync(0xffffffffu, nslots, o);
      if (lane == 0) {
        S.m.q0 = q0;
        S.m.q_rows = q_rows;
        S.m.T = (nslots + BN - 1) / BN;
        S.m.nseg = rp1 - rp0;
        S.m.kv_row0 = (int)(((long long)b * p.Hkv + hq / p.G) * p.L);
        S.m.q_row0 = (int)(((long long)b * p.Hq + hq) * p.L);
        S.m.rp0 = rp0;
        S.m.b = b;
        S.m.i = i;
        S.m.c_start = c_start;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_SLFULL + sl));
    }
  } else if (warp == W_KPROD || warp == W_VPROD) {
    // ============================================================ producers
    // Both warps walk the same key stream; warp 0 loads Q and K and writes
    // each tile's slot mask and causal description, warp 3 loads V.
    const bool kprod = warp == W_KPROD;
    uint32_t g = 0;
    int n_local = 0;
    for (;; ++n_local) {
      const int sl = n_local % NSLOT;
      if (!fl.wait(bar(B_SLFULL + sl), (n_local / NSLOT) & 1)) break;
      const ItemMeta M = slots[sl].m;
      if (M.T < 0) break;
      const int2* seg_s = slots[sl].seg;
      const int ms = n_local & 1;
      if (kprod) {
        if (n_local >= 2 && !fl.wait(bar(B_QEMPTY + ms), ((n_local >> 1) - 1) & 1)) break;
        if (lane == 0) {
          mbar_arrive_expect_tx(bar(B_QFULL + ms), kQTile);
          const uint32_t dq = sbase + OFF_Q + ms * kQTile;
          tma_load_2d(dq, &maps.q, bar(B_QFULL + ms), 0, M.q_row0 + M.q0);
          tma_load_2d(dq + kQHalf, &maps.q, bar(B_QFULL + ms), 64, M.q_row0 + M.q0);
        }
      }
      const int32_t* ob = p.off + (long long)M.b * (p.Nmax + 1);
      int gbase = -1, g_s0 = 0, g_len = 0;
      auto desc = [&](int sq) -> int2 {
        if (sq < SEG_CAP) return seg_s[sq];
        const int base = sq & ~31;
        if (base != gbase) {
          gbase = base;
          const int q = base + lane;
          if (q < M.nseg) {
            const int j = p.col_idx[M.rp0 + q];
            g_s0 = ob[j];
            g_len = (j == M.i) ? (M.q0 + M.q_rows - M.c_start) : (ob[j + 1] - g_s0);
          }
        }
        return make_int2(__shfl_sync(0xffffffffu, g_s0, sq & 31), __shfl_sync(0xffffffffu, g_len, sq & 31));
      };
      int sq = 0, seg_pos = 0;
      bool ok = true;
      for (int kt = 0; kt < M.T; ++kt, ++g) {
        const int stk = g % NSK, stv = g % NSV, tk = g % NTOK;
        if (kprod) {
          if (g >= NSK && !fl.wait(bar(B_SFULL + (g - NSK) % NSB), ((g - NSK) / NSB) & 1)) { ok = false; break; }
          if (g >= NTOK && !fl.wait(bar(B_TOKEMPTY + tk), ((g / NTOK) - 1) & 1)) { ok = false; break; }
        } else {
          if (g >= NSV && !fl.wait(bar(B_PVDONE + (g - NSV) % NSB), ((g - NSV) / NSB) & 1)) { ok = false; break; }
        }
        int slot = 0, causal = 0, d_slot = 0, d_off = 0, nbox = 0, my_y = 0, my_so = 0, my_bx = 0;
        uint32_t mk0 = 0, mk1 = 0, mk2 = 0, mk3 = 0;
        uint32_t bytes = 0;
        while (slot < BN && sq < M.nseg) {
          const int2 dsc = desc(sq);
          const int rows = min(dsc.y - seg_pos, BN - slot);
          const int groups = (rows + 7) >> 3;
          const int tok0 = dsc.x + seg_pos;
          if (kprod) {
            mk0 |= mask_bits(slot, slot + rows, 0);
            mk1 |= mask_bits(slot, slot + rows, 1);
            mk2 |= mask_bits(slot, slot + rows, 2);
            mk3 |= mask_bits(slot, slot + rows, 3);
            if (sq == M.nseg - 1 && tok0 + rows - 1 > M.q0) {
              causal = 1;
              d_slot = slot;
              d_off = slot - tok0;
            }
          }
          if (lane == nbox) {
            my_y = M.kv_row0 + tok0;
            my_so = slot * 128;
            my_bx = groups - 1;
          }
          bytes += (uint32_t)groups * 8u * 256u;
          ++nbox;
          slot += groups * 8;
          seg_pos += rows;
          if (seg_pos == dsc.y) {
            seg_pos = 0;
            ++sq;
          }
        }
        if (kprod) {
          if (lane == 0) {
            TileInfo& ti = tile_info[tk];
            ti.mask[0] = mk0;
            ti.mask[1] = mk1;
            ti.mask[2] = mk2;
            ti.mask[3] = mk3;
            ti.causal = causal;
            ti.d_slot = d_slot;
            ti.d_off = d_off;
            mbar_arrive(bar(B_TOKFULL + tk));
            mbar_arrive_expect_tx(bar(B_KFULL + stk), bytes);
          }
          __syncwarp();
          const uint32_t dk = sbase + OFF_K + stk * kKTile;
          if (lane < nbox) {
            tma_load_2d(dk + my_so, &maps.k[my_bx], bar(B_KFULL + stk), 0, my_y);
            tma_load_2d(dk + kKHalf + my_so, &maps.k[my_bx], bar(B_KFULL + stk), 64, my_y);
          }
        } else {
          if (lane == 0) mbar_arrive_expect_tx(bar(B_VFULL + stv), bytes);
          __syncwarp();
          const uint32_t dv = sbase + OFF_V + stv * kKTile;
          if (lane < nbox) {
            tma_load_2d(dv + my_so, &maps.v[my_bx], bar(B_VFULL + stv), 0, my_y);
            tma_load_2d(dv + kKHalf + my_so, &maps.v[my_bx], bar(B_VFULL + stv), 64, my_y);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_SLEMPTY + sl));
      if (!ok) break;
    }
    // drain: every copy this warp issued must have landed before teardown
    if (lane == 0) {
      if (kprod) {
        for (uint32_t gg = (g > NSK ? g - NSK : 0); gg < g; ++gg)
          mbar_wait(bar(B_KFULL + gg % NSK), (gg / NSK) & 1, kWaitLimitNs);
        for (int n = (n_local > 2 ? n_local - 2 : 0); n < n_local; ++n)
          mbar_wait(bar(B_QFULL + (n & 1)), (n >> 1) & 1, kWaitLimitNs);
      } else {
        for (uint32_t gg = (g > NSV ? g - NSV : 0); gg < g; ++gg)
          mbar_wait(bar(B_VFULL + gg % NSV), (gg / NSV) & 1, kWaitLimitNs);
      }
    }
  } else if (warp == W_QK) {
    // ============================================================ S^T issuer
    // S^T[g % NSB] = K(g) Q^T: M = 128 key slots, N = 64 query rows. The
    // buffer is reused once the softmax has read S^T(g - NSB).
    if (lane == 0) {
      const uint32_t idesc_qk = idesc_tr(BN, NQ, false, false);
      uint32_t g = 0;
      int n_local = 0;
      for (;; ++n_local) {
        const int sl = n_local % NSLOT;
        if (!fl.wait(bar(B_SLFULL + sl), (n_local / NSLOT) & 1)) break;
        const int T = slots[sl].m.T;
        if (T < 0) break;
        mbar_arrive(bar(B_SLEMPTY + sl));
        const int ms = n_local & 1;
        if (!fl.wait(bar(B_QFULL + ms), (n_local >> 1) & 1)) break;
        const uint32_t qa = sbase + OFF_Q + ms * kQTile;
        bool ok = true;
        for (int kt = 0; kt < T; ++kt, ++g) {
          const int stk = g % NSK, sb = g % NSB;
          if (!fl.wait(bar(B_KFULL + stk), (g / NSK) & 1)) { ok = false; break; }
          if (g >= NSB && !fl.wait(bar(B_SREAD + sb), ((g / NSB) - 1) & 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t k0 = sbase + OFF_K + stk * kKTile;
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            mma_ss(tmem + sb * NQ, smem_desc_sw128(k0 + (ks >> 2) * kKHalf + (ks & 3) * 32, 16, 1024),
                   smem_desc_sw128(qa + (ks >> 2) * kQHalf + (ks & 3) * 32, 16, 1024), idesc_qk, ks > 0 ? 1u : 0u);
          mma_commit(bar(B_SFULL + sb));
          if (kt == T - 1) mma_commit(bar(B_QEMPTY + ms));
        }
        if (!ok) break;
        if (T == 0) mma_commit(bar(B_QEMPTY + ms));
      }
      mma_commit(bar(B_FINAL));
      mbar_wait(bar(B_FINAL), 0, kWaitLimitNs);
    }
  } else if (warp == W_PV) {
    // ============================================================ O^T issuer
    // O^T += V^T(g) P^T(g): A = V^T (head-dim contiguous in the V tile),
    // B = P^T (query contiguous, written by the softmax warps).
    if (lane == 0) {
      const uint32_t idesc_pv = idesc_tr(128, NQ, true, true);
      const uint32_t tO = tmem + kTmemO;
      uint32_t g = 0;
      int n_local = 0;
      for (;; ++n_local) {
        const int sl = n_local % NSLOT;
        if (!fl.wait(bar(B_SLFULL + sl), (n_local / NSLOT) & 1)) break;
        const int T = slots[sl].m.T;
        if (T < 0) break;
        mbar_arrive(bar(B_SLEMPTY + sl));
        // the item's first MMA overwrites O^T: the previous epilogue must have read it
        if (n_local > 0 && !fl.wait(bar(B_EPIDONE), (n_local - 1) & 1)) break;
        bool ok = true;
        for (int kt = 0; kt < T; ++kt, ++g) {
          const int stv = g % NSV, sb = g % NSB;
          if (!fl.wait(bar(B_PREADY + sb), (g / NSB) & 1)) { ok = false; break; }
          if (!fl.wait(bar(B_VFULL + stv), (g / NSV) & 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t v0 = sbase + OFF_V + stv * kKTile, p0 = sbase + OFF_P + sb * kPTile;
#pragma unroll
          for (int ks = 0; ks < BN / 16; ++ks)
            mma_ss(tO, smem_desc_sw128(v0 + ks * 2048, kKHalf, 1024), smem_desc_sw128(p0 + ks * 2048, kKHalf, 1024),
                   idesc_pv, (kt > 0 || ks > 0) ? 1u : 0u);
          mma_commit(bar(B_PVDONE + sb));
          if (kt == T - 1) mma_commit(bar(B_OFINAL));
        }
        if (!ok) break;
        if (T == 0) mma_commit(bar(B_OFINAL));
      }
      mma_commit(bar(B_FINALPV));
      mbar_wait(bar(B_FINALPV), 0, kWaitLimitNs);
    }
  } else if (warp >= W_SOFTMAX0 && warp < W_SOFTMAX0 + kSoftmaxWarps) {
    // ============================================================ softmax + epilogue
    const int quarter = warp & 3;               // TMEM lanes 32*quarter .. +31
    const int half = (warp - W_SOFTMAX0) >> 2;  // query columns 32*half .. +31
    const int gbar = 1 + half;                  // this warpgroup's named barrier
    regs_inc<kRegsSoftmax>();
    const int slot = quarter * 32 + lane;       // key slot = TMEM lane (= head-dim row of O^T)
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_addr + half * 32;
    const uint32_t tO = tmem + lane_addr + kTmemO + half * 32;
    float* nm_s = reinterpret_cast<float*>(smem + OFF_NM) + half * 64;         // [buffer][32]
    unsigned* red = reinterpret_cast<unsigned*>(smem + OFF_RED) + half * 128;   // [quarter][32]
    float* lred = reinterpret_cast<float*>(smem + OFF_LRED) + half * 128;       // [quarter][32]
    const float c = p.scale_log2;
    uint32_t g = 0;
    int n_local = 0, cur = 0;
    bool ok = true;
    for (;; ++n_local) {
      const int sl = n_local % NSLOT;
      const bool got = fl.wait(bar(B_SLFULL + sl), (n_local / NSLOT) & 1);
      if (group_any(gbar, !got)) break;
      const ItemMeta M = slots[sl].m;
      if (M.T < 0) break;                  // end of the work list (the same slot for the whole group)
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_SLEMPTY + sl));
      float l[32];                         // partial row sums of this slot, per query column
#pragma unroll
      for (int e = 0; e < 32; ++e) l[e] = 0.f;
      bool stop = false;
      for (int kt = 0; kt < M.T; ++kt, ++g) {
        const int sb = g % NSB, tk = g % NTOK;
        bool okt = fl.wait(bar(B_SFULL + sb), (g / NSB) & 1) && fl.wait(bar(B_TOKFULL + tk), (g / NTOK) & 1);
        // the P^T buffer is free once the MMA of tile g - NSB has completed
        okt = okt && (g < NSB || fl.wait(bar(B_PVDONE + sb), ((g / NSB) - 1) & 1));
        okt = __all_sync(0xffffffffu, okt) && ok;
        uint32_t s[32];
        uint32_t mw = 0;
        int causal = 0, d_slot = 0, d_off = 0;
        if (okt) {
          tc_fence_after();
          tmem_ld32(tS + sb * NQ, s);
          tmem_wait_ld();
          const TileInfo& ti = tile_info[tk];
          mw = ti.mask[quarter];
          causal = ti.causal;
          d_slot = ti.d_slot;
          d_off = ti.d_off;
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) s[e] = 0u;
        }
        // columns e < thr of this half do not see this slot (padding, or a
        // key after the query in the diagonal chunk)
        int thr = 0;
        if (!((mw >> lane) & 1u)) thr = 32;
        else if (causal && slot >= d_slot) thr = slot - d_off - M.q0 - 32 * half;
        // x = s c - m, with nm = -m in shared memory (+inf: no key seen yet)
        float x[32];
        const float4* nm4 = reinterpret_cast<const float4*>(nm_s + cur * 32);
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
          const float4 n = nm4[e4];
          x[4 * e4 + 0] = fmaf(__uint_as_float(s[4 * e4 + 0]), c, n.x);
          x[4 * e4 + 1] = fmaf(__uint_as_float(s[4 * e4 + 1]), c, n.y);
          x[4 * e4 + 2] = fmaf(__uint_as_float(s[4 * e4 + 2]), c, n.z);
          x[4 * e4 + 3] = fmaf(__uint_as_float(s[4 * e4 + 3]), c, n.w);
        }
#pragma unroll
        for (int e = 0; e < 32; ++e)
          if (e < thr) x[e] = -INFINITY;
        float xm[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
          xm[q] = max3(max3(x[q], x[q + 4], x[q + 8]), max3(x[q + 12], x[q + 16], x[q + 20]), fmaxf(x[q + 24], x[q + 28]));
        const bool need = kt == 0 || fmaxf(fmaxf(xm[0], xm[1]), fmaxf(xm[2], xm[3])) > kRaise;
        if (group_any(gbar, need || !okt)) {
          // ---- the rare path: raise the column maxima of this half
          if (group_any(gbar, !okt)) {
            stop = true;
            break;
          }
          // the scores again (S^T is only released below), so that the
          // common path need not keep them
          tmem_ld32(tS + sb * NQ, s);
          tmem_wait_ld();
          unsigned mine = 0;   // lane e: this warp's max key of column e
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const unsigned k = warp_max_u32(fkey(e < thr ? -INFINITY : __uint_as_float(s[e])));
            if (lane == e) mine = k;
          }
          red[quarter * 32 + lane] = mine;
          group_sync(gbar);
          // new maxima: quarter 0 publishes column `lane`'s; every thread
          // derives the rescale factors (the same in all threads)
          const float nm_old_l = kt == 0 ? INFINITY : nm_s[cur * 32 + lane];
          if (quarter == 0) {
            const unsigned kl = max(max(red[lane], red[32 + lane]), max(red[64 + lane], red[96 + lane]));
            const float m_new = fmaxf(-nm_old_l, unfkey(kl) * c);
            nm_s[(cur ^ 1) * 32 + lane] = m_new == -INFINITY ? INFINITY : -m_new;
          }
          float f[32];
          bool rescale = false;
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4) {
            const float4 n = kt == 0 ? make_float4(INFINITY, INFINITY, INFINITY, INFINITY) : nm4[e4];
            const uint4 r0 = reinterpret_cast<const uint4*>(red)[e4], r1 = reinterpret_cast<const uint4*>(red + 32)[e4];
            const uint4 r2 = reinterpret_cast<const uint4*>(red + 64)[e4], r3 = reinterpret_cast<const uint4*>(red + 96)[e4];
            const unsigned kk[4] = {max(max(r0.x, r1.x), max(r2.x, r3.x)), max(max(r0.y, r1.y), max(r2.y, r3.y)),
                                    max(max(r0.z, r1.z), max(r2.z, r3.z)), max(max(r0.w, r1.w), max(r2.w, r3.w))};
            const float nn[4] = {n.x, n.y, n.z, n.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int e = 4 * e4 + j;
              const float m_old = -nn[j];
              const float m_new = fmaxf(m_old, unfkey(kk[j]) * c);
              f[e] = m_new == m_old ? 1.f : fast_exp2(m_old - m_new);
              rescale |= f[e] != 1.f;
              l[e] *= f[e];
            }
          }
          // O^T columns follow the new maxima (the branch is uniform); the
          // MMA of the previous tile must have completed
          if (kt > 0 && rescale) {
            bool okr = fl.wait(bar(B_PVDONE + (g - 1) % NSB), ((g - 1) / NSB) & 1);
            okr = __all_sync(0xffffffffu, okr);
            if (okr) {
              tc_fence_after();
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                uint32_t o[16];
                tmem_ld16(tO + 16 * h, o);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f[16 * h + e]);
                tmem_st16(tO + 16 * h, o);
              }
              tmem_wait_st();
            }
            ok = ok && okr;    // a failure is acted on at the group's next reduction
          }
          group_sync(gbar);    // the new maxima are visible; red may be rewritten
          cur ^= 1;
          const float4* nn4 = reinterpret_cast<const float4*>(nm_s + cur * 32);
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4) {
            const float4 n = nn4[e4];
            x[4 * e4 + 0] = fmaf(__uint_as_float(s[4 * e4 + 0]), c, n.x);
            x[4 * e4 + 1] = fmaf(__uint_as_float(s[4 * e4 + 1]), c, n.y);
            x[4 * e4 + 2] = fmaf(__uint_as_float(s[4 * e4 + 2]), c, n.z);
            x[4 * e4 + 3] = fmaf(__uint_as_float(s[4 * e4 + 3]), c, n.w);
          }
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (e < thr) x[e] = -INFINITY;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(bar(B_SREAD + sb));
          mbar_arrive(bar(B_TOKEMPTY + tk));
        }
        // P^T row of this slot: 32 bf16 (this half's columns), 128-byte swizzle
        uint32_t pk[16];
#pragma unroll
        for (int cc = 0; cc < 16; ++cc) {
          const float p0 = fast_exp2(x[2 * cc]), p1 = fast_exp2(x[2 * cc + 1]);
          l[2 * cc] += p0;
          l[2 * cc + 1] += p1;
          pk[cc] = pack_bf16x2(p0, p1);
        }
        unsigned char* prow = smem + OFF_P + sb * kPTile + slot * 128;
#pragma unroll
        for (int jj = 0; jj < 4; ++jj)
          *reinterpret_cast<uint4*>(prow + (((4 * half + jj) ^ (slot & 7)) << 4)) =
              make_uint4(pk[4 * jj], pk[4 * jj + 1], pk[4 * jj + 2], pk[4 * jj + 3]);
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_PREADY + sb));
      }
      if (stop) break;
      // ---- epilogue: O = O^T / l, written as bf16 (an empty key set, which
      // valid CSR input never has, writes zeros)
      const bool oko = fl.wait(bar(B_OFINAL), n_local & 1);
      if (group_any(gbar, !(oko && ok))) break;
      // reduce-scatter of the row sums over the warp's 32 slots: lane e ends
      // with column e
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) {
        const bool up = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < o; ++i) {
          const float send = up ? l[i] : l[i + o];
          const float keep = up ? l[i + o] : l[i];
          l[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
      }
      lred[quarter * 32 + lane] = l[0];
      group_sync(gbar);
      float inv[32];
#pragma unroll
      for (int e4 = 0; e4 < 8; ++e4) {
        const float4 a = reinterpret_cast<const float4*>(lred)[e4], b = reinterpret_cast<const float4*>(lred + 32)[e4];
        const float4 d = reinterpret_cast<const float4*>(lred + 64)[e4], h = reinterpret_cast<const float4*>(lred + 96)[e4];
        const float t[4] = {(a.x + b.x) + (d.x + h.x), (a.y + b.y) + (d.y + h.y), (a.z + b.z) + (d.z + h.z),
                            (a.w + b.w) + (d.w + h.w)};
#pragma unroll
        for (int j = 0; j < 4; ++j) inv[4 * e4 + j] = t[j] > 0.f ? 1.f / t[j] : 0.f;
      }
      tc_fence_after();
      uint32_t o[32];
      tmem_ld32(tO, o);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_EPIDONE));   // O^T may be overwritten by the next item
      // thread = head-dim index: each store instruction of the warp writes 32
      // consecutive bf16 of one output row
      __nv_bfloat16* ocol = p.O + ((long long)M.q_row0 + M.q0 + 32 * half) * kHeadDim + slot;
#pragma unroll
      for (int e = 0; e < 32; ++e)
        if (32 * half + e < M.q_rows)
          ocol[(long long)e * kHeadDim] = __float2bfloat16_rn(inv[e] == 0.f ? 0.f : __uint_as_float(o[e]) * inv[e]);
      group_sync(gbar);    // lred may be rewritten
    }
  }

  // ---------------------------------------------------------------- teardown
  __syncwarp();
  tc_fence_before();
  if (warp != W_QK) {
    if (lane == 0) mbar_arrive(bar(B_TEARDOWN));
    return;
  }
  mbar_wait(bar(B_TEARDOWN), 0, kWaitLimitNs);
  __syncwarp();
  tc_fence_after();
  tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

// Launches the persistent kernel over the short work list (built beforehand
// on the same stream). Returns DHSA_OK or the launch error.
int launch_sparse_attn_short(const AttnWork& w, const void* Q, const void* K, const void* V, int B, int Hq, int Hkv,
                             int L, const int32_t* off, int Nmax, const int32_t* row_ptr, const int32_t* col_idx,
                             float softmax_scale, void* O, unsigned int* status, cudaStream_t stream) {
  if (w.cap_short == 0) return DHSA_OK;
  EncodeTiledFn enc = tmap_encode_fn();
  if (!enc) return cuda_status(cudaErrorNotSupported);
  ShortMaps maps;
  const long long q_rows = (long long)B * Hq * L, kv_rows = (long long)B * Hkv * L;
  bool ok = make_rows_map(enc, &maps.q, Q, q_rows, NQ);
  for (int s = 0; s < 16; ++s) {
    ok = ok && make_rows_map(enc, &maps.k[s], K, kv_rows, 8 * (s + 1));
    ok = ok && make_rows_map(enc, &maps.v[s], V, kv_rows, 8 * (s + 1));
  }
  if (!ok) return DHSA_ERR_INVALID_ARG;

  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(sparse_attn_short_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemAlloc);
  if (e != cudaSuccess) return cuda_status(e);

  ShortParams prm;
  prm.off = off;
  prm.row_ptr = row_ptr;
  prm.col_idx = col_idx;
  prm.items = w.items_short;
  prm.n_items = w.n_short;
  prm.work_counter = w.counter_short;
  prm.O = static_cast<__nv_bfloat16*>(O);
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.G = Hq / Hkv;
  prm.L = L;
  prm.Nmax = Nmax;
  prm.scale_log2 = softmax_scale * 1.4426950408889634f;
  prm.status = status;
  const int grid = (int)(w.cap_short < sms ? w.cap_short : sms);
  sparse_attn_short_kernel<<<grid, kThreads, kSmemAlloc, stream>>>(maps, prm);
  return launch_status();
}

}  // namespace dhsa

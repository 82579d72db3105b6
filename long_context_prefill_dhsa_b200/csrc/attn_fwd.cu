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
//   A persistent grid (one CTA per SM) takes items from a work list
//   dynamically (an atomic counter, read by each CTA's scheduler warp); the
//   other roles follow the scheduler's ring.
// * Key stream: the kept chunks of row (b, hq, i) are concatenated and packed
//   into 128-slot key tiles. Each chunk starts on an 8-slot boundary (one
//   128-byte-swizzle atom = 8 rows x 128 B, so every TMA destination is
//   1024-byte aligned) and each piece of a chunk inside a tile is fetched with
//   a single TMA box per head-dim half (16 tensor maps, box heights 8..128
//   rows) at an arbitrary row coordinate: a TMA op has a fixed cost of tens
//   of cycles, so splitting pieces into small boxes starves the pipeline.
// * Masking: padding slots are removed inside the tensor core. Every QK^T
//   gets one extra K=16 MMA step, ones-column x per-slot bias (0 for a kept
//   key, -inf for a padding slot), so S already holds -inf there. Only tiles
//   that hold keys of the diagonal chunk mask causally: that chunk is the
//   key stream's last and its slots hold consecutive tokens, so a row masks
//   the slots from one threshold on. Every chunk takes round8(length)
//   consecutive stream slots, so the scheduler gives the diagonal chunk's
//   first slot with the item and the softmax computes each row's threshold
//   itself.
// * Warp roles (512 threads, four warpgroups): warp 0 = TMA producer of Q
//   and K (and of the bias blocks), warp 3 = TMA producer of V, warp 1 =
//   QK^T issuer, warp 14 = PV issuer (one thread each), warp 2 = scheduler
//   (resolves each work item's chunk list into a shared-memory ring up to 4
//   items ahead), warps 4-11 = softmax + epilogue: two warps per TMEM lane
//   quarter, each owning 16 of its 32 query rows with all 128 key slots of a
//   tile (TMEM shape 16x256b: four threads per row, two rows per thread).
//   Tile row r sits in TMEM lane 32 (r mod 4) + r / 4 (Q is loaded through
//   four views of every fourth row), so the valid rows of a partly filled
//   tile spread over all four lane quarters; a warp whose 16 rows are all
//   past the chunk's end only keeps the barrier counts, and its
//   sub-partition's other warp runs alone.
//   Warpgroups 0 and 3
//   hand their registers to the softmax warpgroups (setmaxnreg). The two
//   issuers sit on sub-partitions apart from the K producer: an issuer that
//   shares one with the K producer measurably slows that sub-partition's
//   softmax warps.
// * Pipelines: Q double-buffered; separate K and V rings of 2 stages; a K
//   stage is released as soon as its QK^T completes, a V stage after its PV.
//   The producers walk a tile's key stream in registers before they wait for
//   its stage, so the copies go out right after the wait (the K stage's
//   barrier gets its byte count first and the producer's arrive last, after
//   the bias block is written): the K producer is on
//   the kernel's critical path, and a few dozen more instructions per tile
//   there cost several percent.
//   With two issuing threads the tensor pipe keeps work queued while either
//   one waits on a barrier.
// * TMEM (512 columns): three S buffers (3 x 128 fp32 columns) and the O
//   accumulator (128 columns). P (bf16 pairs) is written back into the first
//   64 columns of the S buffer it came from (shape 16x128b, where each
//   thread's packed pairs land on their own lane and column) and consumed
//   from TMEM by the PV MMA (A in TMEM, V as an N-major shared-memory
//   operand). The QK^T issuer runs up to three tiles ahead of the PV.
// * Online softmax in the log2 domain. A row's maximum is the max of its four
//   threads' 32 columns, combined with two shuffles: the two warps of a lane
//   quarter trade nothing per tile. One exponential pair in four is computed
//   on the FMA pipe (exp2_poly2), the rest by the MUFU; the scale and the
//   row sums use packed f32x2 operations. The running max is only raised (and
//   O rescaled in TMEM, each warp its own rows) when it grows by more than 8
//   (a factor 256), which keeps O / l exact while skipping nearly all
//   rescales; only then does the softmax wait for the previous PV. At the
//   end of an item the row sums go through shared memory to the epilogue's
//   32x32b layout, where each warp writes 64 output columns of 32 rows.
// * Every mbarrier wait is bounded; a timeout sets DHSA_DEVFLAG_WAIT_TIMEOUT,
//   the CTA drains its own in-flight copies and MMAs (again bounded), frees
//   its TMEM and exits.
#include <cuda.h>

#include "common.cuh"
#include "sm100_ptx.cuh"
#include "tmap.cuh"

namespace dhsa {
namespace {

using namespace ptx;

constexpr int BM = kQueryTileRows;   // query rows per tile
constexpr int BN = 128;              // key slots per tile
constexpr int NSK = 2;               // K pipeline stages
constexpr int NSV = 2;               // V pipeline stages
constexpr int NSB = 3;               // S/P buffers in TMEM
constexpr int NSLOT = 4;             // scheduled work items in flight
constexpr int SEG_CAP = 64;          // chunk descriptors kept in shared memory per item
constexpr int kThreads = 512;
constexpr uint32_t kHalfBytes = 128 * 128;   // 128 rows x 64 bf16 (one 128B-swizzled half tile)
constexpr uint32_t kTileBytes = 2 * kHalfBytes;
constexpr uint32_t kBiasBytes = 128 * 16 * 2;  // 128 rows x 16 bf16, no swizzle
constexpr uint32_t kTmemCols = 512;
constexpr uint16_t kBf16One = 0x3F80, kBf16NegInf = 0xFF80;

struct AttnMaps {
  CUtensorMap q[4];   // rows r, r+4, r+8, ... of Q (r = 0..3), box 64 x 32 rows
  CUtensorMap k[16];  // boxes 64 cols x 8*(n+1) rows: one TMA per chunk piece and head-dim half
  CUtensorMap v[16];
};

struct AttnParams {
  const int32_t* off;
  const int32_t* row_ptr;
  const int32_t* col_idx;
  const int4* items;      // (b, hq, i, tile)
  const int* n_items;
  int* work_counter;      // next unassigned item (zeroed by the work-list builder)
  __nv_bfloat16* O;
  int Hq, Hkv, G, L, Nmax;
  float scale_log2;
  unsigned int* status;
  unsigned long long wait_limit_ns;   // limit of the pipeline waits (1 s)
  int hold_scheduler;                 // test hook: publish no item, so the first waits run out
};

// One scheduled work item, written by the scheduler warp.
struct ItemMeta {
  int q0;        // token of the first query row
  int q_rows;    // valid query rows (1..128)
  int T;         // key tiles
  int nseg;      // kept chunks (the last one is the diagonal chunk)
  int kv_row0;   // global K/V row of token 0 of this (b, kv head)
  int q_row0;    // global Q/O row of token 0 of this (b, q head)
  int rp0;       // first CSR entry of the row
  int b;
  int i;         // query chunk
  int c_start;   // first token of chunk i
  int diag_slot; // key-stream slot where the diagonal chunk starts
  int pad;
};
struct ItemSlot {
  ItemMeta m;
  int2 seg[SEG_CAP];   // (first token, visible length) of the first SEG_CAP kept chunks
};

// shared-memory layout (offsets from a 1024-aligned base)
constexpr uint32_t OFF_Q = 0;                                   // 2 x 32 KB
constexpr uint32_t OFF_K = OFF_Q + 2 * kTileBytes;              // NSK x 32 KB
constexpr uint32_t OFF_V = OFF_K + NSK * kTileBytes;            // NSV x 32 KB
constexpr uint32_t OFF_ONES = OFF_V + NSV * kTileBytes;         // 4 KB
constexpr uint32_t OFF_BIAS = OFF_ONES + kBiasBytes;            // NSK x 4 KB
constexpr uint32_t OFF_SLOT = OFF_BIAS + NSK * kBiasBytes;
constexpr uint32_t OFF_XCHG = OFF_SLOT + NSLOT * sizeof(ItemSlot);   // row sums, [item parity][row]
constexpr uint32_t OFF_BAR = OFF_XCHG + 2 * BM * 4;
enum {
  B_QFULL = 0,
  B_QEMPTY = B_QFULL + 2,
  B_SLFULL = B_QEMPTY + 2,
  B_SLEMPTY = B_SLFULL + NSLOT,
  B_KFULL = B_SLEMPTY + NSLOT,
  B_VFULL = B_KFULL + NSK,
  B_SFULL = B_VFULL + NSV,   // QK^T(g) complete: S ready, K stage and bias block free
  B_PREADY = B_SFULL + NSB,
  B_PVDONE = B_PREADY + NSB,     // PV(g) complete: P buffer and V stage free, O current
  B_OFINAL = B_PVDONE + NSB,
  B_FINAL = B_OFINAL + 1,
  B_FINALPV = B_FINAL + 1,
  B_XSUM = B_FINALPV + 1,        // [quarter][item parity]: the softmax pair's row-sum hand-over
  B_TEARDOWN = B_XSUM + 8,
  B_COUNT = B_TEARDOWN + 1
};
constexpr uint32_t OFF_TMEMPTR = OFF_BAR + 8 * B_COUNT;
constexpr uint32_t OFF_ABORT = OFF_TMEMPTR + 4;
constexpr uint32_t kSmemBytes = OFF_ABORT + 4;
constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;  // slack for aligning the base
static_assert(kSmemAlloc <= 227 * 1024, "shared memory budget");
static_assert(OFF_BAR % 8 == 0 && OFF_SLOT % 16 == 0, "alignment");

// role warps
constexpr int W_PRODUCER = 0, W_MMA = 1, W_SCHED = 2, W_VPRODUCER = 3, W_SOFTMAX0 = 4, W_PV = 14;
constexpr int kSoftmaxWarps = 8;
constexpr int kSlotConsumers = 2 + 2 + kSoftmaxWarps;  // K and V producers, QK and PV issuers, softmax warps
// registers per thread after reallocation: warpgroup 0 (producers, scheduler,
// QK issuer) and warpgroup 3 (PV issuer) give theirs to the two softmax
// warpgroups
constexpr uint32_t kRegsLaunch = 65536 / kThreads / 8 * 8;   // 128 at 512 threads
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

// pairs of fp32 in one 64-bit register, for the packed f32x2 operations
__device__ __forceinline__ uint64_t pk2(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void unpk2(uint64_t v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// 2^x of two values on the FMA pipe, so that the special-function unit is
// not the only source of the softmax's exponentials. x = j + f with
// j = round(x), taken by adding 1.5 * 2^23 (the integer lands in the low
// mantissa bits of the sum) and |f| <= 1/2; 2^f = 1 + f (c1 + f (c2 + f c3)),
// the coefficients minimising the maximum relative error on [-1/2, 1/2]
// (exp2_poly.py beside this file fits them; 1.01e-4, twenty times below
// bf16's rounding step); j is added into the exponent field. x = 0 gives
// exactly 1. Inputs are clamped at -127, where j = -127 and f = 0 make the
// sum's bits exactly +0: masked scores (-inf) give P = 0 as the MUFU does.
// On (-127, -126) the result lies in [0, 2^-126); for j = -127, f >= 0, so
// the exponent field never borrows into the sign.
constexpr float kExpC1 = 0.69328302f, kExpC2 = 0.24221103f, kExpC3 = 0.05500864f;
__device__ __forceinline__ void exp2_poly2(uint64_t x2, float& p0, float& p1) {
  float x0, x1;
  unpk2(x2, x0, x1);
  x2 = pk2(fmaxf(x0, -127.f), fmaxf(x1, -127.f));
  const uint64_t t = add2(x2, pk2(12582912.f, 12582912.f));
  const uint64_t j = add2(t, pk2(-12582912.f, -12582912.f));
  const uint64_t f = fma2(j, pk2(-1.f, -1.f), x2);   // exact
  uint64_t q = fma2(pk2(kExpC3, kExpC3), f, pk2(kExpC2, kExpC2));
  q = fma2(q, f, pk2(kExpC1, kExpC1));
  q = fma2(q, f, pk2(1.f, 1.f));
  float q0, q1, t0, t1;
  unpk2(q, q0, q1);
  unpk2(t, t0, t1);
  p0 = __int_as_float(__float_as_int(q0) + (__float_as_int(t0) << 23));
  p1 = __int_as_float(__float_as_int(q1) + (__float_as_int(t1) << 23));
}
// one pair of exponentials in this many goes to exp2_poly2 (measured: 1/4 and
// 1/3 are fastest, 1/2 overloads the FMA pipe, none leaves the MUFU the bound)
constexpr int kPolyPairEvery = 4;

__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// byte offset of element (row, k) in a 128 x 16 bf16 K-major block without swizzle
__device__ __forceinline__ uint32_t noswz_off(int row, int k) {
  return (uint32_t)((row >> 3) * 256 + (k >> 3) * 128 + (row & 7) * 16 + (k & 7) * 2);
}

struct Flags {
  volatile int* abort;
  unsigned int* status;
  unsigned long long limit_ns;
  // The lanes of a warp that wait together poll the same barrier in lockstep
  // and give up together; before giving up the barrier is tested once more,
  // so a phase that completes at the limit still counts. (Making the result
  // warp-uniform with a vote after every wait cost about 5% of the kernel's
  // time: its per-tile chain is that latency-sensitive.)
  __device__ __forceinline__ bool wait(uint32_t bar, uint32_t parity) {
    if (mbar_test_wait(bar, parity)) return true;   // fast path: already complete
    if (*abort) return false;
    if (mbar_wait_slow(bar, parity, limit_ns)) return true;
    if (mbar_test_wait(bar, parity)) return true;
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
  ItemSlot* slots = reinterpret_cast<ItemSlot*>(smem + OFF_SLOT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_ABORT);
  auto bar = [&](int idx) { return sbase + OFF_BAR + 8u * idx; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_items = *p.n_items;

  // ---------------------------------------------------------------- setup
  if (warp == W_PRODUCER) {
    if (lane == 0) {
      *abort_flag = 0;
      for (int s = 0; s < 2; ++s) {
        mbar_init(bar(B_QFULL + s), 1);
        mbar_init(bar(B_QEMPTY + s), 1);
      }
      for (int s = 0; s < NSB; ++s) {
        mbar_init(bar(B_SFULL + s), 1);
        mbar_init(bar(B_PREADY + s), kSoftmaxWarps);
        mbar_init(bar(B_PVDONE + s), 1);
      }
      for (int s = 0; s < NSLOT; ++s) {
        mbar_init(bar(B_SLFULL + s), 1);
        mbar_init(bar(B_SLEMPTY + s), kSlotConsumers);
      }
      for (int s = 0; s < NSK; ++s) mbar_init(bar(B_KFULL + s), 1);
      for (int s = 0; s < NSV; ++s) mbar_init(bar(B_VFULL + s), 1);
      mbar_init(bar(B_OFINAL), 1);
      mbar_init(bar(B_FINAL), 1);
      mbar_init(bar(B_FINALPV), 1);
      for (int s = 0; s < 8; ++s) mbar_init(bar(B_XSUM + s), 2);
      mbar_init(bar(B_TEARDOWN), kThreads / 32 - 1);
      fence_mbar_init();
      for (int r = 0; r < 4; ++r) prefetch_tmap(&maps.q[r]);
      for (int s = 0; s < 16; ++s) {
        prefetch_tmap(&maps.k[s]);
        prefetch_tmap(&maps.v[s]);
      }
    }
  } else if (warp == W_MMA) {
    tmem_alloc(sbase + OFF_TMEMPTR, kTmemCols);
    tmem_relinquish();
  }
  // Slots that no TMA fills in a tile must hold finite values (their logits
  // get -inf added; a masked V row is multiplied by P = 0): zero every K and
  // V stage and the bias blocks once; then write the ones column of the bias
  // step's A operand.
  for (uint32_t o = threadIdx.x * 16; o < OFF_SLOT - OFF_K; o += kThreads * 16)
    *reinterpret_cast<uint4*>(smem + OFF_K + o) = make_uint4(0, 0, 0, 0);
  __syncthreads();
  if (threadIdx.x < BM) *reinterpret_cast<uint16_t*>(smem + OFF_ONES + noswz_off(threadIdx.x, 0)) = kBf16One;
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + OFF_TMEMPTR);
  Flags fl{abort_flag, p.status, p.wait_limit_ns};
  if (warp < W_SOFTMAX0) regs_dec<kRegsWg0>();
  else if (warp >= W_SOFTMAX0 + kSoftmaxWarps) regs_dec<kRegsWg3>();

  if (warp == W_SCHED) {
    // ============================================================ scheduler
    // items are handed out dynamically: the next free item of the list goes
    // to whichever CTA's scheduler asks first; T = -1 marks the end
    int n_local = 0;
    if (p.hold_scheduler) {
      // test hook: publish nothing; the other roles' first waits run out and
      // raise the abort flag before any copy or MMA is issued
      const uint64_t t0 = globaltimer_ns();
      while (!*abort_flag && globaltimer_ns() - t0 < kWaitLimitNs) __nanosleep(1000);
      n_local = -1;
    }
    for (; n_local >= 0; ++n_local) {
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
      const int b = wi.x, hq = wi.y, i = wi.z, tq = wi.w;
      const int32_t* ob = p.off + (long long)b * (p.Nmax + 1);
      const int c_start = ob[i], c_end = ob[i + 1];
      const int q0 = c_start + BM * tq;
      const int q_rows = min(BM, c_end - q0);
      const long long r = ((long long)b * p.Hq + hq) * p.Nmax + i;
      const int rp0 = p.row_ptr[r], rp1 = p.row_ptr[r + 1];
      ItemSlot& S = slots[sl];
      // every chunk takes round8(len) consecutive key-stream slots (a piece
      // split at a tile boundary continues at slot 0 of the next tile)
      int nslots = 0, last = 0;
      for (int q = rp0 + lane; q < rp1; q += 32) {
        const int j = min(max(p.col_idx[q], 0), i);   // a bad index cannot leave the offsets row
        const int s0 = ob[j];
        const int len = (j == i) ? (q0 + q_rows - c_start) : (ob[j + 1] - s0);
        nslots += round8(len);
        if (q == rp1 - 1) last = round8(len);
        if (q - rp0 < SEG_CAP) S.seg[q - rp0] = make_int2(s0, len);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        nslots += __shfl_xor_sync(0xffffffffu, nslots, o);
        last += __shfl_xor_sync(0xffffffffu, last, o);
      }
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
        S.m.diag_slot = nslots - last;   // the diagonal chunk is the row's last
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_SLFULL + sl));
    }
  } else if (warp == W_PRODUCER || warp == W_VPRODUCER) {
    // ============================================================ producers
    // Two warps walk the same key stream: warp 0 loads Q and K (and writes
    // each K stage's bias block), warp 3 loads V. A K
    // stage frees when its QK^T completes and a V stage when its PV does;
    // with separate warps the K loads never wait behind a V stage.
    const bool kprod = warp == W_PRODUCER;
    uint32_t g = 0;  // global key-tile counter of this CTA
    int n_local = 0;
    for (;; ++n_local) {
      const int sl = n_local % NSLOT;
      if (!fl.wait(bar(B_SLFULL + sl), (n_local / NSLOT) & 1)) break;
      const ItemMeta M = slots[sl].m;
      if (M.T < 0) break;                  // end of the work list
      const int2* seg_s = slots[sl].seg;
      const int ms = n_local & 1;
      if (kprod) {
        if (n_local >= 2 && !fl.wait(bar(B_QEMPTY + ms), ((n_local >> 1) - 1) & 1)) break;
        // tile row r goes to TMEM lane 32 (r mod 4) + r / 4: lane q loads
        // rows q, q + 4, ..., q + 124 into the 32 rows of lane quarter q
        if (lane == 0) mbar_arrive_expect_tx(bar(B_QFULL + ms), kTileBytes);
        __syncwarp();
        if (lane < 4) {
          const long long G = (long long)M.q_row0 + M.q0 + lane;
          const CUtensorMap* mq = &maps.q[G & 3];
          const uint32_t dq = sbase + OFF_Q + ms * kTileBytes + lane * 4096;
          tma_load_2d(dq, mq, bar(B_QFULL + ms), 0, (int)(G >> 2));
          tma_load_2d(dq + kHalfBytes, mq, bar(B_QFULL + ms), 64, (int)(G >> 2));
        }
      }
      const int32_t* ob = p.off + (long long)M.b * (p.Nmax + 1);
      // chunk descriptors beyond SEG_CAP are read from global memory, 32 at a time
      int gbase = -1, g_s0 = 0, g_len = 0;
      auto desc = [&](int sq) -> int2 {
        if (sq < SEG_CAP) return seg_s[sq];
        const int base = sq & ~31;
        if (base != gbase) {
          gbase = base;
          const int q = base + lane;
          if (q < M.nseg) {
            const int j = min(max(p.col_idx[M.rp0 + q], 0), M.i);
            g_s0 = ob[j];
            g_len = (j == M.i) ? (M.q0 + M.q_rows - M.c_start) : (ob[j + 1] - g_s0);
          }
        }
        return make_int2(__shfl_sync(0xffffffffu, g_s0, sq & 31), __shfl_sync(0xffffffffu, g_len, sq & 31));
      };
      int sq = 0, seg_pos = 0;
      bool ok = true;
      for (int kt = 0; kt < M.T; ++kt, ++g) {
        const int stk = g % NSK, stv = g % NSV;
        // walk the key stream of this tile first, in registers only (the
        // stage waits below then overlap it): lane b holds the b-th TMA box,
        // and bit i of kept the state of slot lane + 32 i
        int slot = 0, nbox = 0, my_y = 0, my_so = 0, my_bx = 0;
        uint32_t bytes = 0, kept = 0;
        while (slot < BN && sq < M.nseg) {
          const int2 dsc = desc(sq);
          const int rows = min(dsc.y - seg_pos, BN - slot);
          const int groups = (rows + 7) >> 3;
          const int tok0 = dsc.x + seg_pos;
          if (kprod) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int s = lane + 32 * q;
              if (s >= slot && s < slot + rows) kept |= 1u << q;
            }

          }
          // the whole piece in one box per head-dim half (per-op TMA cost
          // dominates for small boxes, so never split a piece)
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
          // the K stage (and its bias block) of tile g - NSK is free once that QK^T is done
          if (g >= NSK && !fl.wait(bar(B_SFULL + (g - NSK) % NSB), ((g - NSK) / NSB) & 1)) { ok = false; break; }
          // copies first; the bias block follows, and the stage's barrier
          // completes only after this warp's arrive
          if (lane == 0) mbar_expect_tx(bar(B_KFULL + stk), bytes);
          __syncwarp();
          const uint32_t dk = sbase + OFF_K + stk * kTileBytes;
          if (lane < nbox) {
            tma_load_2d(dk + my_so, &maps.k[my_bx], bar(B_KFULL + stk), 0, my_y);
            tma_load_2d(dk + kHalfBytes + my_so, &maps.k[my_bx], bar(B_KFULL + stk), 64, my_y);
          }
          unsigned char* bias = smem + OFF_BIAS + stk * kBiasBytes;
#pragma unroll
          for (int q = 0; q < 4; ++q)
            *reinterpret_cast<uint16_t*>(bias + noswz_off(lane + 32 * q, 0)) = ((kept >> q) & 1u) ? 0 : kBf16NegInf;
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(bar(B_KFULL + stk));
          }
        } else {
          // the V stage of tile g - NSV is free once that PV is done
          if (g >= NSV && !fl.wait(bar(B_PVDONE + (g - NSV) % NSB), ((g - NSV) / NSB) & 1)) { ok = false; break; }
          if (lane == 0) mbar_arrive_expect_tx(bar(B_VFULL + stv), bytes);
          __syncwarp();
          const uint32_t dv = sbase + OFF_V + stv * kTileBytes;
          if (lane < nbox) {
            tma_load_2d(dv + my_so, &maps.v[my_bx], bar(B_VFULL + stv), 0, my_y);
            tma_load_2d(dv + kHalfBytes + my_so, &maps.v[my_bx], bar(B_VFULL + stv), 64, my_y);
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
  } else if (warp == W_MMA) {
    // ============================================================ QK^T issuer
    // S[g % NSB] = Q K(g)^T (+ ones x bias). The buffer last held P(g - NSB),
    // so it is reused once PV(g - NSB) has completed.
    if (lane == 0) {
      const uint32_t idesc_qk = idesc_bf16_f32(BM, BN, false);
      const uint32_t tS0 = tmem;
      const uint64_t ones_desc = smem_desc_noswz(sbase + OFF_ONES, 128, 256);
      uint32_t g = 0;
      int n_local = 0;
      for (;; ++n_local) {
        const int sl = n_local % NSLOT;
        if (!fl.wait(bar(B_SLFULL + sl), (n_local / NSLOT) & 1)) break;
        const int T = slots[sl].m.T;
        if (T < 0) break;                  // end of the work list
        mbar_arrive(bar(B_SLEMPTY + sl));
        const int ms = n_local & 1;
        if (!fl.wait(bar(B_QFULL + ms), (n_local >> 1) & 1)) break;
        const uint32_t qa = sbase + OFF_Q + ms * kTileBytes;
        bool ok = true;
        for (int kt = 0; kt < T; ++kt, ++g) {
          const int stk = g % NSK, sb = g % NSB;
          if (!fl.wait(bar(B_KFULL + stk), (g / NSK) & 1)) { ok = false; break; }
          if (g >= NSB && !fl.wait(bar(B_PVDONE + sb), ((g / NSB) - 1) & 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t k0 = sbase + OFF_K + stk * kTileBytes;
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const uint32_t ko = (ks >> 2) * kHalfBytes + (ks & 3) * 32;
            mma_ss(tS0 + sb * 128, smem_desc_sw128(qa + ko, 16, 1024), smem_desc_sw128(k0 + ko, 16, 1024),
                   idesc_qk, ks > 0 ? 1u : 0u);
          }
          // S += ones x bias: -inf on padding slots
          mma_ss(tS0 + sb * 128, ones_desc, smem_desc_noswz(sbase + OFF_BIAS + stk * kBiasBytes, 128, 256),
                 idesc_qk, 1u);
          mma_commit(bar(B_SFULL + sb));
          if (kt == T - 1) mma_commit(bar(B_QEMPTY + ms));
        }
        if (!ok) break;
        if (T == 0) mma_commit(bar(B_QEMPTY + ms));   // an empty key set: nothing to multiply
      }
      // drain this thread's tensor work before TMEM is released
      mma_commit(bar(B_FINAL));
      mbar_wait(bar(B_FINAL), 0, kWaitLimitNs);
    }
  } else if (warp == W_PV) {
    // ============================================================ PV issuer
    // O += P(g) V(g), P read from TMEM where the softmax left it. A second
    // issuing thread keeps the tensor pipe fed while the QK^T issuer waits.
    if (lane == 0) {
      const uint32_t idesc_pv = idesc_bf16_f32(BM, 128, true);
      const uint32_t tS0 = tmem, tO = tmem + 384;
      uint32_t g = 0;
      int n_local = 0;
      for (;; ++n_local) {
        const int sl = n_local % NSLOT;
        if (!fl.wait(bar(B_SLFULL + sl), (n_local / NSLOT) & 1)) break;
        const int T = slots[sl].m.T;
        if (T < 0) break;                  // end of the work list
        mbar_arrive(bar(B_SLEMPTY + sl));
        bool ok = true;
        for (int kt = 0; kt < T; ++kt, ++g) {
          const int stv = g % NSV, sb = g % NSB;
          if (!fl.wait(bar(B_PREADY + sb), (g / NSB) & 1)) { ok = false; break; }
          if (!fl.wait(bar(B_VFULL + stv), (g / NSV) & 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t v0 = sbase + OFF_V + stv * kTileBytes;
#pragma unroll
          for (int ks = 0; ks < BN / 16; ++ks) {
            const uint64_t bdesc = smem_desc_sw128(v0 + ks * 2048, kHalfBytes, 1024);
            // P of key slots 16ks .. 16ks + 15 sits in S columns 8ks .. 8ks + 7
            mma_ts(tO, tS0 + sb * 128 + ks * 8, bdesc, idesc_pv,
                   (kt > 0 || ks > 0) ? 1u : 0u);
          }
          mma_commit(bar(B_PVDONE + sb));
          if (kt == T - 1) mma_commit(bar(B_OFINAL));
        }
        if (!ok) break;
        if (T == 0) mma_commit(bar(B_OFINAL));
      }
      mma_commit(bar(B_FINALPV));
      mbar_wait(bar(B_FINALPV), 0, kWaitLimitNs);
    }
  } else if (warp >= W_SOFTMAX0 && warp < W_SOFTMAX0 + 8) {
    // ============================================================ softmax + epilogue
    // Two warps per TMEM lane quarter, each owning 16 of its 32 query rows
    // with all 128 key slots of every tile. TMEM shape 16x256b: thread t holds
    // rows t/4 and t/4 + 8 of the warp's 16, 32 columns of each; the four
    // threads of a row combine their maxima with two shuffles, so the warps
    // trade nothing per tile and need not run in step.
    const int quarter = warp & 3;             // TMEM lanes 32*quarter .. +31
    const int half = (warp - W_SOFTMAX0) >> 2;
    regs_inc<kRegsSoftmax>();
    const int cq = lane & 3;
    // TMEM lane 32q + l holds query row 4l + q of the tile
    const int tlA = quarter * 32 + half * 16 + (lane >> 2), tlB = tlA + 8;     // TMEM lanes of the two rows
    const int rowA = 4 * (tlA - quarter * 32) + quarter, rowB = rowA + 32;   // query rows within the tile
    const uint32_t tS0 = tmem + ((uint32_t)(quarter * 32 + half * 16) << 16);
    const uint32_t tO16 = tS0 + 384;
    // epilogue: 32x32b, thread = TMEM lane quarter*32 + lane (query row
    // 4 lane + quarter), O columns half*64 .. +63
    const int row = 4 * lane + quarter;
    const uint32_t tO = tmem + ((uint32_t)(quarter * 32) << 16) + 384 + half * 64;
    float* xsum = reinterpret_cast<float*>(smem + OFF_XCHG);    // [item parity][row]
    const float c = p.scale_log2;
    const uint64_t c2 = pk2(c, c);
    uint32_t g = 0;
    int n_local = 0;
    for (;; ++n_local) {
      const int sl = n_local % NSLOT;
      if (!fl.wait(bar(B_SLFULL + sl), (n_local / NSLOT) & 1)) break;
      const ItemMeta M = slots[sl].m;
      if (M.T < 0) break;                  // end of the work list
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_SLEMPTY + sl));
      const int qtA = M.q0 + rowA, qtB = M.q0 + rowB;
      // a warp whose 16 rows are all past the chunk's end does no softmax work
      // (the P of its lanes only feeds O rows that are never stored)
      const bool idle = 64 * half + quarter >= M.q_rows;
      float mA = -INFINITY, mB = -INFINITY, lA = 0.f, lB = 0.f;
      bool ok = true;
      for (int kt = 0; kt < M.T; ++kt, ++g) {
        const int sb = g % NSB;
        if (idle) {
          // S(g) complete implies PREADY's phase of tile g - NSB completed, so
          // this arrive counts toward tile g
          if (!fl.wait(bar(B_SFULL + sb), (g / NSB) & 1)) {
            ok = false;
            break;
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(B_PREADY + sb));
          continue;
        }
        if (!fl.wait(bar(B_SFULL + sb), (g / NSB) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // s[4j + e]: row A, column 8j + 2cq + e; s[4j + 2 + e]: row B, same column
        uint32_t s[64];
        tmem_ld_16x256b_x8(tS0 + sb * 128 + 0, *reinterpret_cast<uint32_t(*)[32]>(s + 0));
        tmem_ld_16x256b_x8(tS0 + sb * 128 + 64, *reinterpret_cast<uint32_t(*)[32]>(s + 32));
        tmem_wait_ld();
        // the diagonal chunk, the key stream's last, starts at slot dt of this
        // tile (dt < 0: in an earlier tile) and its slot s holds token
        // c_start + s - dt: a row masks the slots from qt - c_start + dt + 1 on
        const int dt = M.diag_slot - BN * kt;
        if (dt < BN) {
          const int thrA = max(qtA - M.c_start + dt + 1, 0), thrB = max(qtB - M.c_start + dt + 1, 0);
#pragma unroll
          for (int j = 0; j < 16; ++j)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int col = 8 * j + 2 * cq + e;
              if (col >= thrA) s[4 * j + e] = __float_as_uint(-INFINITY);
              if (col >= thrB) s[4 * j + 2 + e] = __float_as_uint(-INFINITY);
            }
        }
        // row maxima: two chains per row over the thread's 32 columns
        auto S = [&](int e) { return __uint_as_float(s[e]); };
        float a0 = fmaxf(S(0), S(1)), a1 = fmaxf(S(4), S(5));
        float b0 = fmaxf(S(2), S(3)), b1 = fmaxf(S(6), S(7));
#pragma unroll
        for (int j = 2; j < 16; j += 2) {
          a0 = max3(a0, S(4 * j), S(4 * j + 1));
          a1 = max3(a1, S(4 * j + 4), S(4 * j + 5));
          b0 = max3(b0, S(4 * j + 2), S(4 * j + 3));
          b1 = max3(b1, S(4 * j + 6), S(4 * j + 7));
        }
        float xA = fmaxf(a0, a1), xB = fmaxf(b0, b1);
        xA = fmaxf(xA, __shfl_xor_sync(0xffffffffu, xA, 1));
        xB = fmaxf(xB, __shfl_xor_sync(0xffffffffu, xB, 1));
        xA = fmaxf(xA, __shfl_xor_sync(0xffffffffu, xA, 2));
        xB = fmaxf(xB, __shfl_xor_sync(0xffffffffu, xB, 2));
        const float nA = fmaxf(mA, xA * c), nB = fmaxf(mB, xB * c);
        const bool rA = nA > mA + 8.0f, rB = nB > mB + 8.0f;   // also true on the first tile
        if (kt > 0 && __any_sync(0xffffffffu, rA || rB)) {
          // O may only be touched once the previous tile's PV has finished
          if (!fl.wait(bar(B_PVDONE + (g - 1) % NSB), ((g - 1) / NSB) & 1)) { ok = false; break; }
          tc_fence_after();
          const float fA = rA ? fast_exp2(mA - nA) : 1.f, fB = rB ? fast_exp2(mB - nB) : 1.f;
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            uint32_t o[16];
            tmem_ld_16x256b_x4(tO16 + 32 * c4, o);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              o[4 * j + 0] = __float_as_uint(__uint_as_float(o[4 * j + 0]) * fA);
              o[4 * j + 1] = __float_as_uint(__uint_as_float(o[4 * j + 1]) * fA);
              o[4 * j + 2] = __float_as_uint(__uint_as_float(o[4 * j + 2]) * fB);
              o[4 * j + 3] = __float_as_uint(__uint_as_float(o[4 * j + 3]) * fB);
            }
            tmem_st_16x256b_x4(tO16 + 32 * c4, o);
          }
          tmem_wait_st();
          if (rA) lA *= fA;
          if (rB) lB *= fB;
        }
        if (rA) mA = nA;
        if (rB) mB = nB;
        // a row whose keys so far are all masked keeps m = -inf: its p are 0
        const uint64_t nA2 = pk2(mA == -INFINITY ? 0.f : -mA, mA == -INFINITY ? 0.f : -mA);
        const uint64_t nB2 = pk2(mB == -INFINITY ? 0.f : -mB, mB == -INFINITY ? 0.f : -mB);
        uint64_t rsA[2] = {0ull, 0ull}, rsB[2] = {0ull, 0ull};
        // two halves of 8 column groups; pk[2u]: P of row A, key slots
        // 16j + 4cq + {0..3} (j = 8h + u) packed as bf16 pairs at column
        // 4j + cq (16x128b: thread t writes lane t/4 from pk[2u] and lane
        // t/4 + 8 from pk[2u + 1])
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t pk[16];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int j = 8 * h + u;
            const uint64_t xa = fma2(pk2(__uint_as_float(s[4 * j]), __uint_as_float(s[4 * j + 1])), c2, nA2);
            const uint64_t xb = fma2(pk2(__uint_as_float(s[4 * j + 2]), __uint_as_float(s[4 * j + 3])), c2, nB2);
            float a0, a1, b0, b1;
            if (j % kPolyPairEvery == kPolyPairEvery - 1) {
              exp2_poly2(xa, a0, a1);
              exp2_poly2(xb, b0, b1);
            } else {
              float x0, x1;
              unpk2(xa, x0, x1);
              a0 = fast_exp2(x0);
              a1 = fast_exp2(x1);
              unpk2(xb, x0, x1);
              b0 = fast_exp2(x0);
              b1 = fast_exp2(x1);
            }
            rsA[u & 1] = add2(rsA[u & 1], pk2(a0, a1));
            rsB[u & 1] = add2(rsB[u & 1], pk2(b0, b1));
            pk[2 * u] = pack_bf16x2(a0, a1);
            pk[2 * u + 1] = pack_bf16x2(b0, b1);
          }
          // P (bf16 pairs) over S columns 32h .. 32h + 31
          tmem_st_16x128b_x8(tS0 + sb * 128 + 32 * h, pk);
        }
        {
          float r0, r1;
          unpk2(add2(rsA[0], rsA[1]), r0, r1);
          lA += r0 + r1;
          unpk2(add2(rsB[0], rsB[1]), r0, r1);
          lB += r0 + r1;
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_PREADY + sb));
      }
      if (!ok) break;
      // epilogue: the row sums (four threads per row) go through shared
      // memory to the 32x32b layout; O / l -> bf16, each warp 64 columns of
      // the quarter's 32 rows (an empty key set, which valid CSR input never
      // has, writes zeros)
      lA += __shfl_xor_sync(0xffffffffu, lA, 1);
      lB += __shfl_xor_sync(0xffffffffu, lB, 1);
      lA += __shfl_xor_sync(0xffffffffu, lA, 2);
      lB += __shfl_xor_sync(0xffffffffu, lB, 2);
      const int lb = n_local & 1;
      if (cq == 0) {
        xsum[lb * BM + tlA] = lA;
        xsum[lb * BM + tlB] = lB;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_XSUM + quarter * 2 + lb));
      if (!fl.wait(bar(B_XSUM + quarter * 2 + lb), (n_local >> 1) & 1)) break;
      const float l_tot = xsum[lb * BM + quarter * 32 + lane];
      if (!fl.wait(bar(B_OFINAL), n_local & 1)) break;
      tc_fence_after();
      const float inv_l = M.T > 0 ? 1.f / l_tot : 0.f;
      const int qt = M.q0 + row;
      __nv_bfloat16* orow = p.O + ((long long)M.q_row0 + qt) * kHeadDim + half * 64;
#pragma unroll
      for (int c4 = 0; c4 < 2; ++c4) {
        uint32_t o[32];
        tmem_ld32(tO + 32 * c4, o);
        tmem_wait_ld();
        if (M.T == 0) {
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = 0u;
        }
        if (row < M.q_rows) {
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
    }
  }

  // ---------------------------------------------------------------- teardown
  // Every warp reports to one mbarrier and exits; warp 1, which allocated
  // TMEM, frees it once all the others (and its own MMAs) are done.
  __syncwarp();  // lanes that waited out their role's single-thread work reconverge here
  tc_fence_before();
  if (warp != W_MMA) {
    if (lane == 0) mbar_arrive(bar(B_TEARDOWN));
    return;
  }
  mbar_wait(bar(B_TEARDOWN), 0, kWaitLimitNs);
  __syncwarp();
  tc_fence_after();
  tmem_dealloc(tmem, kTmemCols);
}


}  // namespace

// Launches the persistent kernel over the long work list (built beforehand
// on the same stream). Returns DHSA_OK or the launch error.
int launch_sparse_attn_long(const AttnWork& w, const void* Q, const void* K, const void* V, int B, int Hq, int Hkv,
                            int L, const int32_t* off, int Nmax, const int32_t* row_ptr, const int32_t* col_idx,
                            float softmax_scale, void* O, unsigned int* status, cudaStream_t stream) {
  if (w.cap_long == 0) return DHSA_OK;
  EncodeTiledFn enc = tmap_encode_fn();
  if (!enc) return cuda_status(cudaErrorNotSupported);
  AttnMaps maps;
  const long long q_rows = (long long)B * Hq * L, kv_rows = (long long)B * Hkv * L;
  // Q as four views of every fourth row (residues 0..3); an empty residue
  // class (fewer than four rows in all) reuses view 0
  bool ok = true;
  for (int r = 0; r < 4; ++r) {
    const long long n_r = (q_rows - r + 3) / 4;
    const int src = n_r > 0 ? r : 0;
    ok = ok && make_rows_view_map(enc, &maps.q[r], reinterpret_cast<const __nv_bfloat16*>(Q) + (long long)src * kHeadDim,
                                  n_r > 0 ? n_r : (q_rows + 3) / 4, 4, 32);
  }
  for (int s = 0; s < 16; ++s) {
    ok = ok && make_rows_map(enc, &maps.k[s], K, kv_rows, 8 * (s + 1));
    ok = ok && make_rows_map(enc, &maps.v[s], V, kv_rows, 8 * (s + 1));
  }
  if (!ok) return DHSA_ERR_INVALID_ARG;

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
  prm.items = w.items_long;
  prm.n_items = w.n_long;
  prm.work_counter = w.counter_long;
  prm.O = static_cast<__nv_bfloat16*>(O);
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.G = Hq / Hkv;
  prm.L = L;
  prm.Nmax = Nmax;
  prm.scale_log2 = softmax_scale * 1.4426950408889634f;
  prm.status = status;
  prm.wait_limit_ns = kWaitLimitNs;
  prm.hold_scheduler = 0;
  unsigned long long test_ns = 0;
  if (take_wait_test(1, &test_ns)) {   // test hook: the first waits run out after test_ns
    prm.wait_limit_ns = test_ns;
    prm.hold_scheduler = 1;
  }
  const int grid = (int)(w.cap_long < sms ? w.cap_long : sms);
  sparse_attn_fwd_kernel<<<grid, kThreads, kSmemAlloc, stream>>>(maps, prm);
  return launch_status();
}

}  // namespace dhsa

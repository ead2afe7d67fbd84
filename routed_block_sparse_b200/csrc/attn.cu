// Index-based block-sparse attention over routed 128-token KV tiles.
//
// Digest of arXiv 2610.22311, "Core method" (Eq. 15) and "Novelty"; Velox
// project page, "Why the route is a block, not a token": the kernel visits
// only the KV tiles listed in a query block's route, so a skipped tile saves
// both its QK^T product and its K/V load.  The result is an ordinary softmax
// attention restricted to the tokens of the listed tiles, computed with the
// FlashAttention online-softmax recurrence over tiles.
//
// sm_100a design: one CTA per (head, query block), one CTA per SM, 384
// threads in three warpgroups.  CTAs take rows in the order `row_order`
// gives (longest routes first, from velox_route_schedule), so the last wave
// is made of short rows.
//
// TMEM (512 columns): two S buffers (fp32, 128 columns each), one O
// accumulator (fp32, 128) and two P buffers (bf16 pairs, 64 each).  Tile j
// has its S in buffer j mod 2 and its P in buffer j mod 2; the softmax of
// even and odd tiles runs in two warpgroups at once.  Because P has buffers
// of its own, S_{j+2} can be issued as soon as the softmax of tile j has
// loaded S_j into registers: the score product of a tile overlaps the
// softmax of the tile before it in the same buffer, and the per-buffer chain
// S -> softmax -> PV -> S is broken.
//
// All tiles accumulate into the one O, so all of them use one per-row
// reference max: tile j takes the reference of tile j - 1 (handed over per
// row through shared memory) and raises it only when its own row max exceeds
// it by more than 2^8 (a stale reference is exact: P and the row sums use
// the same one).  When it rises, O is rescaled in TMEM between PV_{j-1} and
// PV_j by the softmax threads of tile j.
//   warpgroup 0 (56 registers per thread after setmaxnreg), one thread per
//   warp active:
//     warp 0    TMA producer of the route's K tiles, warp 2 of its V
//               tiles, into two rings of 32 KB slots (128-byte swizzle, two
//               64-channel boxes per tile): a K slot is freed by its score
//               product, a V slot by its PV, so neither stream waits on the
//               other.
//     warp 1    TMEM allocator and issuer of the score products: S_{j+2} =
//               Q K_{j+2}^T once the softmax of tile j has read S_j.
//     warp 3    issuer of O += P_j V_j (A = P from TMEM, B = V from shared
//               memory) once P_j is written.  Two issuing threads: each
//               tcgen05.commit tracks only its own thread's products, so a
//               PV never waits behind a K load and S never behind a PV.
//   warpgroups 1 and 2 (224 registers per thread): softmax of the even and
//     of the odd tiles, one query row per thread (its TMEM lane): the whole
//     128-column S row read from TMEM in one go, the row max, the reference
//     hand-over, exponent arguments and the row sum in packed fp32x2
//     arithmetic, exponentials on MUFU (a share of them, set by kPolyPairs,
//     by a cubic on the FMA pipe), P packed to bf16 into its P buffer
//     (column t/2 holds elements t, t+1).  Each warpgroup keeps its row sums
//     in the reference of its own last tile; the epilogue brings both to the
//     final reference and writes O / l and the lse.
// A pre-pass compacts the route into shared memory, skipping ids outside
// [0, M) and repeats (flagged in dev_status); Q's load is issued before it.
//
// Two-phase form (digest, "Reproducibility": the two-phase tile loop): after
// the routed history tiles the same loop visits the n_cur tiles of the
// current chunk's own K/V (separate tensors), like any other tiles, so the
// one softmax covers both phases.
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"

// Of every 8 exponent pairs of a row, this many are computed by the cubic on
// the FMA pipe instead of MUFU (0..8).
#ifndef VELOX_ATTN_POLY_PAIRS
#define VELOX_ATTN_POLY_PAIRS 0
#endif

namespace velox {
namespace {

constexpr int BM = 128;  // query rows per tile
constexpr int BN = 128;  // tokens per KV tile
constexpr int D = 128;   // head dim
constexpr int kThreads = 384;       // 3 warpgroups
constexpr int kChainThreads = 128;  // softmax threads of one warpgroup
constexpr int kSoftThreads = 256;
// register split: the launch gives every thread kRegsLaunch; warpgroup 0
// hands registers back and the two softmax warpgroups take them
constexpr int kRegsLaunch = 168;
constexpr int kRegsCtl = 56;
constexpr int kRegsSoft = 224;
static_assert(128 * kRegsCtl + 2 * 128 * kRegsSoft <= kThreads * kRegsLaunch,
              "setmaxnreg split exceeds the registers the block is launched with");
constexpr int kPolyPairs = VELOX_ATTN_POLY_PAIRS;
static_assert(kPolyPairs >= 0 && kPolyPairs <= 8, "kPolyPairs out of range");
constexpr uint32_t kTileBytes = BN * D * 2;      // 32 KB
constexpr uint32_t kHalfBytes = kTileBytes / 2;  // one 64-channel box
constexpr int kMaxRoute = VELOX_MAX_ROUTE;
constexpr uint32_t kTmemCols = 512;
constexpr int kBufs = 2;             // S and P buffers (tile j uses buffer j mod 2)
constexpr uint32_t kColS = 0;        // S buffers: columns 0 and 128
constexpr uint32_t kColO = 256;      // O accumulator: columns 256..383
constexpr uint32_t kColP = 384;      // P buffers: columns 384 and 448
constexpr int kMaxSlots = 6;         // K/V ring slots of 32 KB
constexpr float kRescaleThreshold = 8.0f;  // log2 of the largest tolerated growth

// shared-memory layout (offsets from a 1024-byte aligned base)
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffRing = kOffQ + kTileBytes;
// barriers, misc, the reference hand-over and the route list follow the ring
// (offsets set at launch).  Barriers: q_full, the K/V ring (full, empty),
// per buffer s_full / s_free / p_full / pv_done, x_fin, mma_done.
constexpr uint32_t kNumBars = 1 + 2 * kMaxSlots + 4 * kBufs + 1 + 1;
constexpr uint32_t kMiscBytes = 64;
constexpr uint32_t kRefBytes = BM * 8;  // per row: reference bits, index of the tile that wrote it
constexpr uint32_t kSmemLimit = 227 * 1024;

struct AttnArgs {
  const uint16_t *Q;         // [H][N * 128][128] bf16
  const int32_t *route_ids;  // null: dense
  const int32_t *route_len;
  const int32_t *row_order;  // null: row = blockIdx.x
  int R_max;
  int N, M;
  int rows;                  // H * N
  int n_cur;                 // current-chunk tiles after the routed ones (0: none)
  float scale_log2;  // softmax_scale * log2(e)
  uint16_t *O;
  float *lse;
  int32_t *dev_status;
  int nslot;              // ring slots in use (4 or 6): half K, half V
  uint32_t bar_offset;    // byte offset of the barriers from the aligned base
  uint32_t ref_offset;    // reference hand-over (fp32 per row)
  uint32_t list_offset;   // route list (uint16)
};

__device__ __forceinline__ uint64_t kmajor_desc(uint32_t tile_saddr, int k) {
  // K-major operand, 128-byte swizzle: 16-element K steps advance 32 bytes
  // inside a 64-element atom; atoms (64 channels) are 16 KB apart.
  return smem_desc_sw128(tile_saddr + (k >> 2) * kHalfBytes + (k & 3) * 32, 16, 1024);
}
__device__ __forceinline__ uint64_t vmn_desc(uint32_t tile_saddr, int k) {
  // V as the MN-major B operand (N = channel, K = token): 16-token K steps
  // advance 16 rows of 128 bytes; the two 64-channel halves are 16 KB apart.
  return smem_desc_sw128(tile_saddr + k * 16 * 128, kHalfBytes, 1024);
}

// D[tmem] (+)= A[tmem] * B[smem desc], kind::f16: A (P, bf16) read from TMEM.
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Warp-uniform bounded wait (tcgen05.ld/st after it are warp-collective).
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort));
}

// The per-row reference word: {value bits, tile index}, stored and loaded
// as one 64-bit shared-memory access so the pair is always consistent.
__device__ __forceinline__ void ref_word_store(uint32_t saddr, uint32_t val, uint32_t tag) {
  asm volatile("st.volatile.shared.v2.u32 [%0], {%1, %2};" ::"r"(saddr), "r"(val), "r"(tag)
               : "memory");
}
// Polls the word until it carries `tag`; gives up (false, *abort set) after
// the same time limit as mbar_wait, or when another thread has aborted.
__device__ __forceinline__ bool ref_word_wait(uint32_t saddr, uint32_t tag, volatile int *abort,
                                              float *val) {
  uint64_t t0 = 0;
  for (uint32_t it = 0;; ++it) {
    uint32_t v, t;
    asm volatile("ld.volatile.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v), "=r"(t) : "r"(saddr)
                 : "memory");
    if (t == tag) {
      *val = __uint_as_float(v);
      return true;
    }
    if ((it & 255u) == 255u) {
      if (*abort) return false;
      const uint64_t now = global_timer_ns();
      if (t0 == 0) {
        t0 = now;
      } else if (now - t0 > kWaitLimitNs) {
        *abort = 1;
        return false;
      }
    }
  }
}

// 2^x for a pair of fp32 values on the FMA pipe: x = k + f with k the
// nearest integer (the 1.5 * 2^23 shifter puts k in the low mantissa bits)
// and f in [-0.5, 0.5]; 2^f from a cubic fitted to it here by iterated
// weighted least squares for the smallest relative error on [-0.5, 0.5]
// (7.5e-5, far below the bf16 rounding of P); k is added to the exponent
// field.  Arguments are clamped at -125 so the result stays a normal number
// (2^-125 instead of a smaller value: an absolute error below 3e-38 against
// a row sum of at least 2^-8).
__device__ __forceinline__ uint64_t exp2_poly2(uint64_t x2) {
  constexpr float kShift = 12582912.0f;  // 1.5 * 2^23
  constexpr float c0 = 0.99992806f, c1 = 0.69326097f, c2 = 0.24261114f, c3 = 0.055171669f;
  float a, b;
  f2unpack(x2, a, b);
  const uint64_t x = f2pack(fmaxf(a, -125.0f), fmaxf(b, -125.0f));
  const uint64_t t = fadd2(x, f2pack(kShift, kShift));
  const uint64_t kf = fadd2(t, f2pack(-kShift, -kShift));
  const uint64_t f = ffma2(kf, f2pack(-1.0f, -1.0f), x);
  uint64_t p = ffma2(f2pack(c3, c3), f, f2pack(c2, c2));
  p = ffma2(p, f, f2pack(c1, c1));
  p = ffma2(p, f, f2pack(c0, c0));
  float p0, p1, t0, t1;
  f2unpack(p, p0, p1);
  f2unpack(t, t0, t1);
  const float r0 = __int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23));
  const float r1 = __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23));
  return f2pack(r0, r1);
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKc,
                const __grid_constant__ CUtensorMap tmVc, AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  uint8_t *sQ = base + kOffQ;
  uint8_t *ring = base + kOffRing;
  uint64_t *bar = reinterpret_cast<uint64_t *>(base + a.bar_offset);
  uint64_t *q_full = bar;
  uint64_t *slot_full = q_full + 1;
  uint64_t *slot_empty = slot_full + kMaxSlots;
  uint64_t *s_full = slot_empty + kMaxSlots;  // [buffer]: S_j written
  uint64_t *s_free = s_full + kBufs;          // [buffer]: S_j read by its softmax
  uint64_t *p_full = s_free + kBufs;          // [buffer]: P_j written
  uint64_t *pv_done = p_full + kBufs;         // [buffer]: PV_j (and all before) done
  uint64_t *x_fin = pv_done + kBufs;          // both warpgroups' row sums written
  uint64_t *mma_done = x_fin + 1;             // every MMA of the CTA done
  uint8_t *misc = base + a.bar_offset + kNumBars * 8;
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(misc);
  int *s_nvalid = reinterpret_cast<int *>(misc + 4);
  volatile int *s_abort = reinterpret_cast<volatile int *>(misc + 8);
  uint32_t refx = smem_u32(base + a.ref_offset);  // [row] {reference bits, tile index}
  uint16_t *tiles = reinterpret_cast<uint16_t *>(base + a.list_offset);
  // the id bitmap of the route compaction and the raw route live in the
  // ring, idle until the first load (bitmap: M bits <= 8 KB; route: R_max
  // int32 <= 16 KB after it)
  uint32_t *bits = reinterpret_cast<uint32_t *>(ring);
  int32_t *raw = reinterpret_cast<int32_t *>(ring + 8192);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = a.row_order ? a.row_order[blockIdx.x] : (int)blockIdx.x;
  if (row < 0 || row >= a.rows) {  // same value in every thread: uniform exit
    if (threadIdx.x == 0) flag_error(a.dev_status, VELOX_DEV_BAD_ROW_ORDER);
    return;
  }
  const int h = row / a.N, i = row - h * a.N;
  const bool dense = (a.route_ids == nullptr);
  const int M = a.M;
  const int nslot = a.nslot;

  // ---- set-up: barriers, TMEM, route compaction
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kMaxSlots; ++s) {
      mbar_init(&slot_full[s], 1);
      mbar_init(&slot_empty[s], 1);
    }
    for (int b = 0; b < kBufs; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_free[b], kChainThreads / 32);  // one arrival per warp
      mbar_init(&p_full[b], kChainThreads / 32);
      mbar_init(&pv_done[b], 1);
    }
    mbar_init(x_fin, kSoftThreads);
    mbar_init(mma_done, 2);  // one commit from each MMA-issuing thread
    *s_abort = 0;
    fence_mbar_init();
    // Q does not depend on the route: its load overlaps the compaction
    prefetch_tmap(&tmQ);
    mbar_arrive_expect_tx(q_full, kTileBytes);
    tma_load_3d(sQ, &tmQ, q_full, 0, i * BM, h);
    tma_load_3d(sQ + kHalfBytes, &tmQ, q_full, 64, i * BM, h);
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, kTmemCols);
    tmem_relinquish();
  }
  if (threadIdx.x < BM) ref_word_store(refx + threadIdx.x * 8, 0u, 0xFFFFFFFFu);  // no tile yet
  int L = 0;
  if (!dense) {
    L = a.route_len[row];
    if (L < 0 || L > a.R_max) {
      if (threadIdx.x == 0) flag_error(a.dev_status, VELOX_DEV_ROUTE_LEN);
      L = 0;
    }
    const int W = (M + 31) >> 5;
    for (int k = threadIdx.x; k < W; k += kThreads) bits[k] = 0u;
    // stage the route in shared memory in one parallel pass (one global
    // round trip instead of one per 32 ids in the ordered pass below)
    const int32_t *ids = a.route_ids + (size_t)row * a.R_max;
    for (int k = threadIdx.x; k < L; k += kThreads) raw[k] = ids[k];
  }
  __syncthreads();
  if (warp == 0) {
    if (dense) {
      if (lane == 0) *s_nvalid = M;
    } else {
      int n = 0;
      bool bad = false, dup = false;
      for (int b0 = 0; b0 < L; b0 += 32) {
        const int j = b0 + lane;
        const int id = j < L ? raw[j] : -1;
        bool ok = (j < L) && id >= 0 && id < M;
        if (j < L && !ok) bad = true;
        if (ok) {
          const uint32_t m = 1u << (id & 31);
          if (atomicOr(&bits[id >> 5], m) & m) {
            ok = false;
            dup = true;
          }
        }
        const unsigned vote = __ballot_sync(0xffffffffu, ok);
        if (ok) tiles[n + __popc(vote & ((1u << lane) - 1u))] = static_cast<uint16_t>(id);
        n += __popc(vote);
      }
      if (__any_sync(0xffffffffu, bad) && lane == 0) flag_error(a.dev_status, VELOX_DEV_BAD_ROUTE_ID);
      if (__any_sync(0xffffffffu, dup) && lane == 0) flag_error(a.dev_status, VELOX_DEV_DUP_ROUTE_ID);
      if (lane == 0) *s_nvalid = n;
    }
  }
  tc_fence_before();
  __syncthreads();  // the bitmap is dead from here on: the ring may be loaded
  tc_fence_after();
  const int n_hist = *s_nvalid;
  const int n = n_hist + a.n_cur;  // tiles of both phases
  const uint32_t tmem = *s_tmem;
  const int wg = warp >> 2;

  if (wg == 0) {
    regs_dec<kRegsCtl>();
    // K and V have rings of their own (kk slots each): a K slot is freed by
    // its score product, a V slot by its PV, so K loads run ahead of the
    // score products without waiting for the PVs and the other way round.
    const int kk = nslot / 2;
    if (warp == 0 || warp == 2) {
      // ================= TMA producers: warp 0 K, warp 2 V =================
      const bool is_k = warp == 0;
      if (lane == 0 && n > 0) {
        const CUtensorMap *hist_map = is_k ? &tmK : &tmV;
        const CUtensorMap *cur_map = is_k ? &tmKc : &tmVc;
        prefetch_tmap(hist_map);
        if (a.n_cur > 0) prefetch_tmap(cur_map);
        // the ring held the compaction bitmap (generic-proxy writes) just
        // before these asynchronous copies overwrite it
        fence_proxy_async_smem();
        const int s0 = is_k ? 0 : kk;  // first slot of this ring
        int issued = 0;
        for (int j = 0; j < n; ++j) {
          const int s = s0 + j % kk;
          const uint32_t use = j / kk;
          if (!mbar_wait(&slot_empty[s], (use & 1) ^ 1, s_abort)) break;
          const bool hist = j < n_hist;
          const int tile = hist ? (dense ? j : tiles[j]) : j - n_hist;
          const CUtensorMap *map = hist ? hist_map : cur_map;
          uint8_t *dst = ring + s * kTileBytes;
          mbar_arrive_expect_tx(&slot_full[s], kTileBytes);
          tma_load_3d(dst, map, &slot_full[s], 0, tile * BN, h);
          tma_load_3d(dst + kHalfBytes, map, &slot_full[s], 64, tile * BN, h);
          issued = j + 1;
        }
        if (*s_abort) {
          // let the copies already in flight land before the CTA goes away
          // (each wait is bounded by the same time limit)
          volatile int never = 0;
          if (is_k) mbar_wait(q_full, 0, &never);
          for (int j = issued - kk < 0 ? 0 : issued - kk; j < issued; ++j) {
            never = 0;
            mbar_wait(&slot_full[s0 + j % kk], (j / kk) & 1, &never);
          }
        }
      }
    } else {
      // ========== MMA issuers: warp 1 the score products, warp 3 the PVs ==========
      // Each thread commits only its own products, so S_{j+2} never waits
      // behind a PV and a PV never waits behind a K load; mma_done takes one
      // arrival from each.
      const bool is_s = warp == 1;
      if (lane == 0 && n > 0) {
        const uint32_t ra = smem_u32(ring);
        bool ok = true;
        if (is_s) {
          constexpr uint32_t idS = idesc_bf16_f32(BM, BN, false);
          const uint32_t qa = smem_u32(sQ);
          // S_j = Q K_j^T into S buffer j mod 2
          auto issue_s = [&](int j) -> bool {
            const int s = j % kk;
            if (!mbar_wait(&slot_full[s], (j / kk) & 1, s_abort)) return false;
            tc_fence_after();
            const uint32_t ka = ra + s * kTileBytes;
            const uint32_t sbuf = tmem + kColS + (j & 1) * BN;
#pragma unroll
            for (int k = 0; k < D / 16; ++k)
              mma_bf16_ss(sbuf, kmajor_desc(qa, k), kmajor_desc(ka, k), idS, k > 0);
            tc_commit(&s_full[j & 1]);
            tc_commit(&slot_empty[s]);
            return true;
          };
          ok = mbar_wait(q_full, 0, s_abort) && issue_s(0);
          if (ok && n > 1) ok = issue_s(1);
          // S_{j+2} goes into the buffer of S_j once its softmax has read it
          for (int j = 0; ok && j + 2 < n; ++j)
            ok = mbar_wait(&s_free[j & 1], (j >> 1) & 1, s_abort) && issue_s(j + 2);
        } else {
          constexpr uint32_t idPV = idesc_bf16_f32(BM, D, true);
          // O += P_j V_j, P_j in P buffer j mod 2 (A from TMEM)
          for (int j = 0; ok && j < n; ++j) {
            const int b = j & 1, s = kk + j % kk;
            ok = mbar_wait(&p_full[b], (j >> 1) & 1, s_abort) &&
                 mbar_wait(&slot_full[s], (j / kk) & 1, s_abort);
            if (!ok) break;
            tc_fence_after();
            const uint32_t va = ra + s * kTileBytes;
            const uint32_t pb = tmem + kColP + b * (BN / 2);
#pragma unroll
            for (int k = 0; k < BN / 16; ++k)
              mma_bf16_ts(tmem + kColO, pb + k * 8, vmn_desc(va, k), idPV, (j > 0 || k > 0));
            tc_commit(&pv_done[b]);
            tc_commit(&slot_empty[s]);
          }
        }
        // every product this thread issued must be complete before TMEM is
        // released (and before the epilogue reads O and reuses the ring)
        tc_commit(mma_done);
        volatile int never = 0;
        mbar_wait(mma_done, 0, &never);
      }
    }
  } else {
    regs_inc<kRegsSoft>();
    // ================= softmax / epilogue (warpgroups 1, 2) =================
    const int quarter = warp & 3;
    const int ch = wg - 1;              // tiles j with j % 2 == ch
    const int r = quarter * 32 + lane;  // query row within the tile = TMEM lane
    const uint32_t trow = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const uint32_t sb = trow + kColS + ch * BN;        // this warpgroup's S buffer
    const uint32_t pb = trow + kColP + ch * (BN / 2);  // this warpgroup's P buffer
    const uint32_t ob = trow + kColO;                  // the O accumulator
    const float c = a.scale_log2;
    float ref_own = -INFINITY;  // reference of this warpgroup's last tile
    float l = 0.f;              // row sum of this warpgroup's tiles, in ref_own
    bool ok = true;
    for (int j = ch; j < n; j += 2) {
      const uint32_t ph = (j >> 1) & 1;
      if (!warp_wait(&s_full[ch], ph, s_abort)) { ok = false; break; }
      tc_fence_after();
      // the whole S row in registers: one TMEM round trip, then the buffer
      // is free for S_{j+2}
      uint32_t sv[128];
      tmem_ld32(sb, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
      tmem_ld32(sb + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
      tmem_ld32(sb + 64, *reinterpret_cast<uint32_t(*)[32]>(&sv[64]));
      tmem_ld32(sb + 96, *reinterpret_cast<uint32_t(*)[32]>(&sv[96]));
      tmem_wait_ld();
#pragma unroll
      for (int q = 0; q < 4; ++q) reg_fence(*reinterpret_cast<uint32_t(*)[32]>(&sv[32 * q]));
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[ch]);
      float mx[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) mx[q] = -INFINITY;
#pragma unroll
      for (int k = 0; k < 64; ++k)
        mx[k & 7] = fmax3(mx[k & 7], __uint_as_float(sv[2 * k]), __uint_as_float(sv[2 * k + 1]));
      const float mt = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]),
                             fmaxf(mx[6], mx[7])) * c;
      // reference hand-over: the thread of this row in the other warpgroup
      // stores {reference, j - 1} as one 64-bit word once tile j - 1 has its
      // max; this thread polls its own row's word (usually one load).  The
      // word holds j - 2 or j - 1 when tile j reads it: tile j + 1 writes
      // only after reading what tile j writes.  This tile raises the
      // reference only on growth above 2^8.
      float ref_prev = -INFINITY;
      if (j > 0) {
        const bool got = ref_word_wait(refx + r * 8, (uint32_t)(j - 1), s_abort, &ref_prev);
        if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      }
      const bool grow = mt > ref_prev + kRescaleThreshold;  // always on tile 0
      const float ref = grow ? mt : ref_prev;
      if (j + 1 < n) ref_word_store(refx + r * 8, __float_as_uint(ref), (uint32_t)j);
      // P buffer reuse: PV_{j-2} (this buffer's last reader) must be done;
      // that also puts every PV before it behind us
      if (j >= 2 && !warp_wait(&pv_done[ch], ((j - 2) >> 1) & 1, s_abort)) { ok = false; break; }
      // O rescale when the reference grew: after PV_{j-1}, before PV_j
      if (j >= 1 && __any_sync(0xffffffffu, grow)) {
        if (!warp_wait(&pv_done[ch ^ 1], ((j - 1) >> 1) & 1, s_abort)) { ok = false; break; }
        tc_fence_after();
        const float alpha = fast_exp2(ref_prev - ref);  // 1 on rows that kept theirs
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t ov[32];
          tmem_ld32(ob + cc * 32, ov);
          tmem_wait_ld();
          reg_fence(ov);
#pragma unroll
          for (int k = 0; k < 32; ++k) ov[k] = __float_as_uint(__uint_as_float(ov[k]) * alpha);
          tmem_st32(ob + cc * 32, ov);
        }
      }
      // exponentials (arguments and row sum in packed pairs); P_j packed to
      // bf16 into its buffer, 16 columns at a time: column t/2 holds
      // elements t, t+1
      uint64_t sum2[2] = {0ull, 0ull};
      const uint64_t c2 = f2pack(c, c), nr2 = f2pack(-ref, -ref);
#pragma unroll
      for (int qt = 0; qt < 4; ++qt) {
        uint32_t pk[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const int e = qt * 16 + k;  // pair index within the row
          const uint64_t x2 =
              ffma2(f2pack(__uint_as_float(sv[2 * e]), __uint_as_float(sv[2 * e + 1])), c2, nr2);
          uint64_t p2;
          if ((e & 7) < kPolyPairs) {
            p2 = exp2_poly2(x2);
          } else {
            float x0, x1;
            f2unpack(x2, x0, x1);
            p2 = f2pack(fast_exp2(x0), fast_exp2(x1));
          }
          sum2[k & 1] = fadd2(sum2[k & 1], p2);
          float p0, p1;
          f2unpack(p2, p0, p1);
          pk[k] = pack_bf16x2(p0, p1);
        }
        tmem_st16(pb + qt * 16, pk);
      }
      float sa, sb2;
      f2unpack(fadd2(sum2[0], sum2[1]), sa, sb2);
      // this warpgroup's row sum moves to the new reference
      l = l * fast_exp2(ref_own - ref) + (sa + sb2);  // 0 * 0 on the first tile
      ref_own = ref;
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[ch]);
    }
    // epilogue: every MMA must be done before O is read and before the ring
    // (idle from then on) takes the row-sum exchange; mma_done completes once
    // per CTA, so the wait cannot meet an older phase.
    bool have = ok && n > 0;
    if (have && !mbar_wait(mma_done, 0, s_abort)) have = false;
    float *xm = reinterpret_cast<float *>(ring);  // [warpgroup][2][128]: reference, sum
    xm[(ch * 2 + 0) * BM + r] = ref_own;
    xm[(ch * 2 + 1) * BM + r] = l;
    mbar_arrive(x_fin);
    const bool fin_ok = mbar_wait(x_fin, 0, s_abort);
    const float ref_o = xm[((ch ^ 1) * 2 + 0) * BM + r];
    const float l_o = xm[((ch ^ 1) * 2 + 1) * BM + r];
    // O is in the reference of the last tile, the larger of the two
    // (references only grow); a warpgroup without tiles has sum 0
    const float ref_fin = fmaxf(ref_own, ref_o);
    const float w_own = l > 0.f ? fast_exp2(ref_own - ref_fin) : 0.f;
    const float w_o = l_o > 0.f ? fast_exp2(ref_o - ref_fin) : 0.f;
    const float l_row = l * w_own + l_o * w_o;
    // tcgen05.ld is warp-collective: decide once for the whole warp
    const bool good = __all_sync(0xffffffffu, have && fin_ok && !*s_abort);
    tc_fence_after();
    const float inv = good ? 1.0f / l_row : 0.f;
    uint16_t *orow = a.O + ((size_t)row * BM + r) * D + ch * 64;
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      uint32_t o0[16];
      if (good) {
        tmem_ld16(ob + ch * 64 + cc * 16, o0);
        tmem_wait_ld();
        reg_fence(o0);
      } else {
#pragma unroll
        for (int k = 0; k < 16; ++k) o0[k] = 0u;
      }
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        float v[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = __uint_as_float(o0[8 * q + e]) * inv;
        uint4 u;
        u.x = pack_bf16x2(v[0], v[1]);
        u.y = pack_bf16x2(v[2], v[3]);
        u.z = pack_bf16x2(v[4], v[5]);
        u.w = pack_bf16x2(v[6], v[7]);
        *reinterpret_cast<uint4 *>(orow + cc * 16 + q * 8) = u;
      }
    }
    if (a.lse && ch == 0)
      a.lse[(size_t)row * BM + r] =
          good ? (ref_fin + __log2f(l_row)) * 0.69314718055994531f : -INFINITY;
  }

  if (threadIdx.x == 0 && n == 0) {
    // nothing waited for Q: its copy must land before the CTA goes away
    volatile int never = 0;
    mbar_wait(q_full, 0, &never);
  }
  if (*s_abort && threadIdx.x == 0) flag_error(a.dev_status, VELOX_DEV_WAIT_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// [H][rows][128] bf16 as a 3-D map (channel, token, head), 64 x 128 boxes.
bool make_map(CUtensorMap *map, const void *ptr, int rows, int H) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)rows, (cuuint64_t)H};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)rows * D * 2};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

int attn_max_route() { return kMaxRoute; }

cudaError_t launch_attn(const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                        const int32_t *route_ids, const int32_t *route_len,
                        const int32_t *row_order, int R_max, const uint16_t *K_cur,
                        const uint16_t *V_cur, int N_cur, int H, int N, int M,
                        float softmax_scale, uint16_t *O, float *lse, int32_t *dev_status,
                        cudaStream_t stream, bool *map_failed) {
  *map_failed = false;
  CUtensorMap mq, mk, mv, mkc, mvc;
  const bool cur = K_cur != nullptr && N_cur > 0;
  if (!make_map(&mq, Q, N * BM, H) || !make_map(&mk, K, M * BN, H) ||
      !make_map(&mv, V, M * BN, H) ||
      !make_map(&mkc, cur ? K_cur : K, cur ? N_cur * BN : M * BN, H) ||
      !make_map(&mvc, cur ? V_cur : V, cur ? N_cur * BN : M * BN, H)) {
    *map_failed = true;
    return cudaErrorInvalidValue;
  }
  AttnArgs a;
  a.Q = Q;
  a.route_ids = route_ids;
  a.route_len = route_len;
  a.row_order = row_order;
  a.R_max = R_max;
  a.N = N;
  a.M = M;
  a.rows = H * N;
  a.n_cur = cur ? N_cur : 0;
  a.scale_log2 = softmax_scale * 1.4426950408889634f;
  a.O = O;
  a.lse = lse;
  a.dev_status = dev_status;
  // tail after the ring: barriers, misc, the reference hand-over, the route
  // list (uint16).  The compaction bitmap (M bits) lives in the ring.
  const uint32_t list_bytes = route_ids ? ((uint32_t)R_max * 2u + 15u) & ~15u : 0u;
  const uint32_t tail = kNumBars * 8 + kMiscBytes + kRefBytes + list_bytes;
  int nslot = kMaxSlots;
  while (nslot > 4 && kOffRing + nslot * kTileBytes + tail + 1024 > kSmemLimit) --nslot;
  // K and V rings of nslot / 2 slots each
  nslot &= ~1;
  a.nslot = nslot;
  a.bar_offset = kOffRing + nslot * kTileBytes;
  a.ref_offset = a.bar_offset + kNumBars * 8 + kMiscBytes;
  a.list_offset = a.ref_offset + kRefBytes;
  const size_t smem = (size_t)a.list_offset + list_bytes + 1024;  // + alignment slack
  // the compaction's bitmap (first 8 KB) and raw route (after it) fit in the ring
  if (smem > kSmemLimit || (size_t)(M + 31) / 32 * 4 > 8192 ||
      (size_t)nslot * kTileBytes < 8192 + (size_t)R_max * 4)
    return cudaErrorInvalidConfiguration;
  // The setmaxnreg split draws on the registers of the launch: refuse to
  // launch a build whose per-thread count is below the one it was planned for
  // (the softmax warpgroups would wait forever for registers).
  static cudaError_t regs_ok = [] {
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, attn_kernel);
    if (e != cudaSuccess) return e;
    return fa.numRegs * kThreads >= 128 * kRegsCtl + 2 * 128 * kRegsSoft
               ? cudaSuccess
               : cudaErrorInvalidConfiguration;
  }();
  if (regs_ok != cudaSuccess) return regs_ok;
  cudaError_t e = cudaFuncSetAttribute(attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  attn_kernel<<<H * N, kThreads, smem, stream>>>(mq, mk, mv, mkc, mvc, a);
  return cudaGetLastError();
}

}  // namespace velox

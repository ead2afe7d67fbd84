// Index-based block-sparse attention over routed 128-token KV tiles.
//
// Digest of arXiv 2610.22311, "Core method" (Eq. 15) and "Novelty"; Velox
// project page, "Why the route is a block, not a token": the kernel visits
// only the KV tiles listed in a query block's route, so a skipped tile saves
// both its QK^T product and its K/V load.  The result is an ordinary softmax
// attention restricted to the tokens of the listed tiles, computed with the
// FlashAttention online-softmax recurrence over tiles.
//
// sm_100a design: one CTA per (head, query block), one CTA per SM; TMEM holds
// two S buffers (128 columns each), the query tile Q (64 columns of bf16
// pairs, the A operand of S = Q K^T) and the O accumulator, so the score
// product reads only K from shared memory.
// CTAs take rows in the order `row_order` gives (longest routes first, from
// velox_route_schedule), so the last wave is made of short rows.
//   warp 0      TMA producer: K_0, V_0, K_1, V_1, ... of the route into a
//               ring of 32 KB slots (128-byte swizzle, two 64-channel boxes
//               per tile).
//   warp 1      TMEM allocator and the single tcgen05.mma issuer.  S_j =
//               Q K_j^T (A = Q from TMEM, B = K from shared memory) goes into
//               buffer j mod 2; once the softmax of tile j is done it issues
//               O += P_j V_j (A = P from TMEM, B = V from shared memory) and,
//               as soon as that has completed, S_{j+2} into the same buffer,
//               so the score product of tile j+1 runs under the softmax of
//               tile j.
//   warps 2-9   softmax: two threads per query row (the row's TMEM lane, in
//               warps w and w + 4), each owning 64 of the tile's 128
//               columns; at the start each writes its half of the row's Q
//               into TMEM, so every scheduler has two softmax warps to switch
//               between.  One TMEM read of the half row, a three-input max,
//               the two half maxima exchanged through shared memory (an
//               mbarrier per S buffer), scaled exponent arguments and the
//               row sum in packed fp32x2 arithmetic, exponentials on MUFU,
//               P_j packed to bf16 into the first 64 columns of its own S
//               buffer (half h writes columns 32h..32h+31, after both halves
//               have read their S).  The running max is only moved (and O
//               rescaled in TMEM, each half its 64 channels, after waiting
//               for PV_{j-1}) when it grows by more than 2^8; otherwise the
//               stale max is kept, which is exact because O and the row sum
//               always use the same max.  Each half keeps its own partial row
//               sum; the epilogue adds them: O / l -> bf16, lse.
// A pre-pass compacts the route into shared memory, skipping ids outside
// [0, M) and repeats (flagged in dev_status).
//
// Two-phase form (digest, "Reproducibility": the two-phase tile loop): after
// the routed history tiles the same loop visits the n_cur tiles of the
// current chunk's own K/V (separate tensors), under the same online softmax,
// so one normaliser covers both phases.
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"

namespace velox {
namespace {

constexpr int BM = 128;  // query rows per tile
constexpr int BN = 128;  // tokens per KV tile
constexpr int D = 128;   // head dim
constexpr int kThreads = 320;  // TMA warp, MMA warp, 8 softmax warps
constexpr int kSoftThreads = 256;
constexpr uint32_t kTileBytes = BN * D * 2;      // 32 KB
constexpr uint32_t kHalfBytes = kTileBytes / 2;  // one 64-channel box
constexpr int kMaxRoute = VELOX_MAX_ROUTE;
constexpr uint32_t kTmemCols = 512;
constexpr int kSBufs = 2;         // S/P buffers in TMEM, columns 0 and 128
constexpr uint32_t kColQ = 256;   // Q (bf16 pairs, 64 columns)
constexpr uint32_t kColO = 384;   // O accumulator (fp32, 128 columns)
constexpr int kMaxSlots = 6;      // K/V ring slots of 32 KB
constexpr float kRescaleThreshold = 8.0f;  // log2 of the largest tolerated growth

// shared-memory layout (offsets from a 1024-byte aligned base)
constexpr uint32_t kOffRing = 0;
// barriers, misc and the dynamic tail follow the ring (offset set at launch)
constexpr uint32_t kNumBars = 1 + 2 * kMaxSlots + 3 * kSBufs + 1 + kSBufs + 1;
constexpr uint32_t kMiscBytes = 64;
// half-row maxima, rounded up to bf16, in two alternating slots ([2][2][128]
// bf16), then the two partial row sums of the epilogue ([2][128] fp32)
constexpr uint32_t kXchBytes = 2 * 2 * BM * 2 + 2 * BM * 4;
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
  int nslot;              // K/V ring slots in use (4..kMaxSlots)
  uint32_t bar_offset;    // byte offset of the barriers from the aligned base
  uint32_t xch_offset;    // half-row maxima exchange area (bf16 bits)
  uint32_t list_offset;   // route list (uint16)
  uint32_t bits_offset;   // id bitmap (uint32)
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

// bf16 bits of finite x rounded towards +inf.
__device__ __forceinline__ uint16_t bf16_round_up(float x) {
  const uint32_t u = __float_as_uint(x);
  uint32_t hi = u >> 16;
  if ((u & 0xffffu) != 0u && (u >> 31) == 0u) hi += 1u;  // positive: away from 0; negative: toward 0
  return static_cast<uint16_t>(hi);
}

// Warp-uniform bounded wait (tcgen05.ld/st after it are warp-collective).
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort));
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKc,
                const __grid_constant__ CUtensorMap tmVc, AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  uint8_t *ring = base + kOffRing;
  uint64_t *bar = reinterpret_cast<uint64_t *>(base + a.bar_offset);
  uint64_t *q_full = bar;
  uint64_t *slot_full = bar + 1;
  uint64_t *slot_empty = slot_full + kMaxSlots;
  uint64_t *s_full = slot_empty + kMaxSlots;
  uint64_t *p_full = s_full + kSBufs;
  uint64_t *pv_done = p_full + kSBufs;
  uint64_t *mma_done = pv_done + kSBufs;
  uint64_t *x_max = mma_done + 1;   // both half-row maxima of S buffer b written
  uint64_t *x_fin = x_max + kSBufs;  // both partial row sums written
  uint8_t *misc = base + a.bar_offset + kNumBars * 8;
  uint16_t *xch = reinterpret_cast<uint16_t *>(base + a.xch_offset);
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(misc);
  int *s_nvalid = reinterpret_cast<int *>(misc + 4);
  volatile int *s_abort = reinterpret_cast<volatile int *>(misc + 8);
  uint16_t *tiles = reinterpret_cast<uint16_t *>(base + a.list_offset);
  uint32_t *bits = reinterpret_cast<uint32_t *>(base + a.bits_offset);

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
    mbar_init(q_full, kSoftThreads);  // Q written to TMEM by the softmax threads
    for (int s = 0; s < kMaxSlots; ++s) {
      mbar_init(&slot_full[s], 1);
      mbar_init(&slot_empty[s], 1);
    }
    for (int b = 0; b < kSBufs; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], kSoftThreads);
      mbar_init(&pv_done[b], 1);
      mbar_init(&x_max[b], kSoftThreads);
    }
    mbar_init(mma_done, 1);
    mbar_init(x_fin, kSoftThreads);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, kTmemCols);
    tmem_relinquish();
  }
  int L = 0;
  if (!dense) {
    L = a.route_len[row];
    if (L < 0 || L > a.R_max) {
      if (threadIdx.x == 0) flag_error(a.dev_status, VELOX_DEV_ROUTE_LEN);
      L = 0;
    }
    const int W = (M + 31) >> 5;
    for (int k = threadIdx.x; k < W; k += kThreads) bits[k] = 0u;
  }
  __syncthreads();
  if (warp == 0) {
    if (dense) {
      if (lane == 0) *s_nvalid = M;
    } else {
      const int32_t *ids = a.route_ids + (size_t)row * a.R_max;
      int n = 0;
      bool bad = false, dup = false;
      for (int b0 = 0; b0 < L; b0 += 32) {
        const int j = b0 + lane;
        const int id = j < L ? ids[j] : -1;
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
  __syncthreads();
  tc_fence_after();
  const int n_hist = *s_nvalid;
  const int n = n_hist + a.n_cur;  // tiles of both phases
  const uint32_t tmem = *s_tmem;

  if (warp == 0) {
    // ================= TMA producer =================
    if (lane == 0 && n > 0) {
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      if (a.n_cur > 0) {
        prefetch_tmap(&tmKc);
        prefetch_tmap(&tmVc);
      }
      int issued = 0;
      for (int li = 0; li < 2 * n; ++li) {  // load li: K_{li/2} (even) or V_{li/2} (odd)
        const int s = li % nslot;
        const uint32_t use = li / nslot;
        if (!mbar_wait(&slot_empty[s], (use & 1) ^ 1, s_abort)) break;
        const int j = li >> 1;
        const bool hist = j < n_hist;
        const int tile = hist ? (dense ? j : tiles[j]) : j - n_hist;
        const CUtensorMap *map = (li & 1) ? (hist ? &tmV : &tmVc) : (hist ? &tmK : &tmKc);
        uint8_t *dst = ring + s * kTileBytes;
        mbar_arrive_expect_tx(&slot_full[s], kTileBytes);
        tma_load_3d(dst, map, &slot_full[s], 0, tile * BN, h);
        tma_load_3d(dst + kHalfBytes, map, &slot_full[s], 64, tile * BN, h);
        issued = li + 1;
      }
      if (*s_abort) {
        // let the copies already in flight land before the CTA goes away
        // (each wait is bounded by the same time limit)
        volatile int never = 0;
        for (int li = issued - nslot < 0 ? 0 : issued - nslot; li < issued; ++li) {
          never = 0;
          mbar_wait(&slot_full[li % nslot], (li / nslot) & 1, &never);
        }
      }
    }
  } else if (warp == 1) {
    // ================= MMA issuer =================
    if (lane == 0 && n > 0) {
      constexpr uint32_t idS = idesc_bf16_f32(BM, BN, false);
      constexpr uint32_t idPV = idesc_bf16_f32(BM, D, true);
      const uint32_t ra = smem_u32(ring);
      auto issue_s = [&](int j) -> bool {
        const int li = 2 * j, s = li % nslot;
        if (!mbar_wait(&slot_full[s], (li / nslot) & 1, s_abort)) return false;
        tc_fence_after();
        const uint32_t ka = ra + s * kTileBytes;
        const uint32_t sb = tmem + (j % kSBufs) * BN;
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          mma_bf16_ts(sb, tmem + kColQ + k * 8, kmajor_desc(ka, k), idS, k > 0);
        tc_commit(&s_full[j % kSBufs]);
        tc_commit(&slot_empty[s]);
        return true;
      };
      bool ok = mbar_wait(q_full, 0, s_abort);
      if (ok) ok = issue_s(0);
      if (ok && n > 1) ok = issue_s(1);
      for (int j = 0; ok && j < n; ++j) {
        const int b = j % kSBufs;
        if (!mbar_wait(&p_full[b], (j / kSBufs) & 1, s_abort)) break;
        const int li = 2 * j + 1, s = li % nslot;
        if (!mbar_wait(&slot_full[s], (li / nslot) & 1, s_abort)) break;
        tc_fence_after();
        const uint32_t va = ra + s * kTileBytes;
        const uint32_t pb = tmem + b * BN;  // P_j: first 64 columns of its S buffer
#pragma unroll
        for (int k = 0; k < BN / 16; ++k)
          mma_bf16_ts(tmem + kColO, pb + k * 8, vmn_desc(va, k), idPV, (j > 0 || k > 0));
        tc_commit(&pv_done[b]);
        tc_commit(&slot_empty[s]);
        if (j + 2 < n) {
          // S_{j+2} goes into the buffer P_j occupies: PV_j must be done
          if (!mbar_wait(&pv_done[b], (j / kSBufs) & 1, s_abort)) break;
          if (!issue_s(j + 2)) break;
        }
      }
      // all issued MMAs must be complete before TMEM is released
      tc_commit(mma_done);
      volatile int never = 0;
      mbar_wait(mma_done, 0, &never);
    }
  } else {
    // ================= softmax / epilogue (warps 2..9) =================
    const int quarter = warp & 3;
    const int hf = (warp - 2) >> 2;     // which 64 columns of the row
    const int r = quarter * 32 + lane;  // query row within the tile = TMEM lane
    const uint32_t trow = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const float c = a.scale_log2;
    float m_run = -INFINITY, l = 0.f;  // l: this half's partial row sum
    bool ok = true;
    if (n > 0) {
      // this thread's half of Q row r into TMEM: bf16 pairs, element 2c in the
      // low half of column c, as the A operand of S = Q K^T expects
      const uint4 *qsrc = reinterpret_cast<const uint4 *>(
          a.Q + (((size_t)h * a.N + i) * BM + r) * D + hf * 64);
      uint32_t qv[32];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const uint4 v = __ldg(qsrc + q);
        qv[4 * q + 0] = v.x;
        qv[4 * q + 1] = v.y;
        qv[4 * q + 2] = v.z;
        qv[4 * q + 3] = v.w;
      }
      tmem_st32(trow + kColQ + hf * 32, qv);
      tmem_wait_st();
    }
    tc_fence_before();
    mbar_arrive(q_full);
    for (int j = 0; j < n; ++j) {
      const int b = j % kSBufs;
      const uint32_t ph = (j / kSBufs) & 1;
      const uint32_t sb = trow + b * BN;
      if (!warp_wait(&s_full[b], ph, s_abort)) { ok = false; break; }
      tc_fence_after();
      uint32_t sv[64];
      tmem_ld32(sb + hf * 64, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
      tmem_ld32(sb + hf * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
      tmem_wait_ld();
      float mx[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) mx[q] = -INFINITY;
#pragma unroll
      for (int k = 0; k < 32; ++k)
        mx[k & 3] = fmax3(mx[k & 3], __uint_as_float(sv[2 * k]), __uint_as_float(sv[2 * k + 1]));
      // exchange the half maxima, each rounded up to bf16 so that both halves
      // take the same (slightly larger, hence still exact) max; slot j & 1 is
      // free again because the partner read it before arriving for tile j - 1.
      // After this wait both halves have read their S columns, so P may
      // overwrite columns 0..63 of the buffer.
      const uint16_t mh = bf16_round_up(fmaxf(fmax3(mx[0], mx[1], mx[2]), mx[3]));
      xch[((j & 1) * 2 + hf) * BM + r] = mh;
      tc_fence_before();
      mbar_arrive(&x_max[b]);
      if (!warp_wait(&x_max[b], ph, s_abort)) { ok = false; break; }
      tc_fence_after();
      const uint16_t mo = xch[((j & 1) * 2 + (hf ^ 1)) * BM + r];
      const float mt = fmaxf(__uint_as_float(static_cast<uint32_t>(mh) << 16),
                             __uint_as_float(static_cast<uint32_t>(mo) << 16));
      const float m_cand = fmaxf(m_run, mt * c);
      const bool grow = m_cand > m_run + kRescaleThreshold;  // always on the first tile
      const float m_use = grow ? m_cand : m_run;
      const float alpha = fast_exp2(m_run - m_use);  // 1 if kept, 0 on the first tile
      if (j > 0 && __any_sync(0xffffffffu, grow)) {
        // move O to the new max: PV_{j-1} (and every earlier PV) must be done
        const int jp = j - 1;
        if (!warp_wait(&pv_done[jp % kSBufs], (jp / kSBufs) & 1, s_abort)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          uint32_t ov[32];
          const uint32_t oa = trow + kColO + hf * 64 + cc * 32;
          tmem_ld32(oa, ov);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) ov[k] = __float_as_uint(__uint_as_float(ov[k]) * alpha);
          tmem_st32(oa, ov);
        }
      }
      // exponentials (arguments and row sum in packed pairs); P_j into the
      // first 64 columns of its S buffer: column t/2 holds elements t, t+1
      uint64_t sum2[2] = {0ull, 0ull};
      const uint64_t c2 = f2pack(c, c), nm2 = f2pack(-m_use, -m_use);
      uint32_t pk[32];
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        const uint64_t x2 = ffma2(f2pack(__uint_as_float(sv[2 * k]), __uint_as_float(sv[2 * k + 1])),
                                  c2, nm2);
        float x0, x1;
        f2unpack(x2, x0, x1);
        const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
        sum2[k & 1] = fadd2(sum2[k & 1], f2pack(p0, p1));
        pk[k] = pack_bf16x2(p0, p1);
      }
      tmem_st32(sb + hf * 32, pk);
      float sa, sb2;
      f2unpack(fadd2(sum2[0], sum2[1]), sa, sb2);
      tmem_wait_st();
      l = l * alpha + (sa + sb2);
      m_run = m_use;
      tc_fence_before();
      mbar_arrive(&p_full[b]);
    }
    // epilogue: the row sum is the sum of the two halves' partial sums
    uint16_t *orow = a.O + ((size_t)row * BM + r) * D + hf * 64;
    bool have = ok && n > 0;
    if (have) {
      const int jl = n - 1;
      have = mbar_wait(&pv_done[jl % kSBufs], (jl / kSBufs) & 1, s_abort);
    }
    float *lx = reinterpret_cast<float *>(base + a.xch_offset + 2 * 2 * BM * 2);
    lx[hf * BM + r] = l;
    mbar_arrive(x_fin);
    const bool fin = mbar_wait(x_fin, 0, s_abort);
    const float l_row = l + lx[(hf ^ 1) * BM + r];
    // tcgen05.ld is warp-collective: decide once for the whole warp
    const bool good = __all_sync(0xffffffffu, have && fin && !*s_abort);
    tc_fence_after();
    const float inv = good ? 1.0f / l_row : 0.f;
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
      uint32_t ov[32];
      if (good) {
        tmem_ld32(trow + kColO + hf * 64 + cc * 32, ov);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int k = 0; k < 32; ++k) ov[k] = 0u;
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint4 v;
        v.x = pack_bf16x2(__uint_as_float(ov[8 * q + 0]) * inv, __uint_as_float(ov[8 * q + 1]) * inv);
        v.y = pack_bf16x2(__uint_as_float(ov[8 * q + 2]) * inv, __uint_as_float(ov[8 * q + 3]) * inv);
        v.z = pack_bf16x2(__uint_as_float(ov[8 * q + 4]) * inv, __uint_as_float(ov[8 * q + 5]) * inv);
        v.w = pack_bf16x2(__uint_as_float(ov[8 * q + 6]) * inv, __uint_as_float(ov[8 * q + 7]) * inv);
        *reinterpret_cast<uint4 *>(orow + cc * 32 + q * 8) = v;
      }
    }
    if (a.lse && hf == 0)
      a.lse[(size_t)row * BM + r] = good ? (m_run + __log2f(l_row)) * 0.69314718055994531f : -INFINITY;
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
  CUtensorMap mk, mv, mkc, mvc;
  const bool cur = K_cur != nullptr && N_cur > 0;
  if (!make_map(&mk, K, M * BN, H) ||
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
  // tail after the ring: barriers, misc, route list (uint16), id bitmap
  const uint32_t list_bytes = route_ids ? ((uint32_t)R_max * 2u + 15u) & ~15u : 0u;
  const uint32_t bits_bytes = route_ids ? (uint32_t)((M + 31) / 32) * 4u : 0u;
  const uint32_t tail = kNumBars * 8 + kMiscBytes + kXchBytes + list_bytes + bits_bytes;
  int nslot = kMaxSlots;
  while (nslot > 4 && kOffRing + nslot * kTileBytes + tail + 1024 > kSmemLimit) --nslot;
  // loads go K_0, V_0, K_1, V_1, ... round the ring; load li reuses the slot
  // of load li - nslot.  With an odd count K_{j+3} would reuse V_j's slot and
  // could not start before PV_j, just when S_{j+3} is wanted: keep it even.
  nslot &= ~1;
  a.nslot = nslot;
  a.bar_offset = kOffRing + nslot * kTileBytes;
  a.xch_offset = a.bar_offset + kNumBars * 8 + kMiscBytes;
  a.list_offset = a.xch_offset + kXchBytes;
  a.bits_offset = a.list_offset + list_bytes;
  const size_t smem = (size_t)a.bits_offset + bits_bytes + 1024;  // + alignment slack
  if (smem > kSmemLimit) return cudaErrorInvalidConfiguration;
  cudaError_t e = cudaFuncSetAttribute(attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  attn_kernel<<<H * N, kThreads, smem, stream>>>(mk, mv, mkc, mvc, a);
  return cudaGetLastError();
}

}  // namespace velox

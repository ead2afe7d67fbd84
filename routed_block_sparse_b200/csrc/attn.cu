// Index-based block-sparse attention over routed 128-token KV tiles.
//
// Digest of arXiv 2610.22311, "Core method" (Eq. 15) and "Novelty"; Velox
// project page, "Why the route is a block, not a token": the kernel visits
// only the KV tiles listed in a query block's route, so a skipped tile saves
// both its QK^T product and its K/V load.  The result is an ordinary softmax
// attention restricted to the tokens of the listed tiles, computed with the
// FlashAttention online-softmax recurrence over tiles.
//
// sm_100a design, one CTA per (head, query block):
//   warp 0      TMA producer: Q once, then K and V tiles of the route into a
//               2-stage ring (128-byte swizzle, two 64-channel boxes a tile);
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer:
//               S_j = Q K_j^T into one of two TMEM S buffers (issued one tile
//               ahead), O += P_j V_j into the TMEM O accumulator;
//   warps 2-5   softmax: one query row per thread (TMEM lane), online max /
//               sum in the log2 domain, O rescaled in TMEM when the row max
//               grows, P_j written as bf16 into swizzled shared memory as the
//               A operand of the PV product; epilogue O / l -> bf16, lse.
// A pre-pass compacts the route into shared memory, skipping ids outside
// [0, M) and repeats (flagged in dev_status).
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"

namespace velox {
namespace {

constexpr int BM = 128;  // query rows per tile
constexpr int BN = 128;  // tokens per KV tile
constexpr int D = 128;   // head dim
constexpr int NS = 2;    // K/V pipeline stages
constexpr int kThreads = 192;
constexpr uint32_t kTileBytes = BN * D * 2;   // 32 KB
constexpr uint32_t kHalfBytes = kTileBytes / 2;  // one 64-channel box
constexpr int kMaxRoute = 4096;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 256;

// shared-memory layout (offsets from a 1024-byte aligned base)
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kOffQ + kTileBytes;
constexpr uint32_t kOffV = kOffK + NS * kTileBytes;
constexpr uint32_t kOffP = kOffV + NS * kTileBytes;
constexpr uint32_t kOffTiles = kOffP + kTileBytes;                 // uint16 x kMaxRoute
constexpr uint32_t kOffBits = kOffTiles + kMaxRoute * 2;           // uint32 x (MAX_BLOCKS/32)
constexpr uint32_t kOffBar = kOffBits + (VELOX_MAX_BLOCKS / 32) * 4;
constexpr uint32_t kNumBars = 1 + 3 * NS + 2 + 2 + 1 + 1 + 1;
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
constexpr uint32_t kSmemBytes = kOffMisc + 64 + 1024;  // + alignment slack

struct AttnArgs {
  const int32_t *route_ids;  // null: dense
  const int32_t *route_len;
  int R_max;
  int N, M;
  float scale_log2;  // softmax_scale * log2(e)
  uint16_t *O;
  float *lse;
  int32_t *dev_status;
};

struct Bars {
  uint64_t *q_full, *k_full, *v_full, *kv_empty, *s_full, *s_free, *p_full, *o_done, *mma_done;
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

__global__ void __launch_bounds__(kThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  uint8_t *sQ = base + kOffQ;
  uint8_t *sK = base + kOffK;
  uint8_t *sV = base + kOffV;
  uint8_t *sP = base + kOffP;
  uint16_t *tiles = reinterpret_cast<uint16_t *>(base + kOffTiles);
  uint32_t *bits = reinterpret_cast<uint32_t *>(base + kOffBits);
  uint64_t *bar = reinterpret_cast<uint64_t *>(base + kOffBar);
  Bars B;
  B.q_full = bar;
  B.k_full = bar + 1;
  B.v_full = bar + 1 + NS;
  B.kv_empty = bar + 1 + 2 * NS;
  B.s_full = bar + 1 + 3 * NS;
  B.s_free = B.s_full + 2;
  B.p_full = B.s_free + 2;
  B.o_done = B.p_full + 1;
  B.mma_done = B.o_done + 1;
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(base + kOffMisc);
  int *s_nvalid = reinterpret_cast<int *>(base + kOffMisc + 4);
  volatile int *s_abort = reinterpret_cast<volatile int *>(base + kOffMisc + 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x;
  const int h = row / a.N, i = row - h * a.N;
  const bool dense = (a.route_ids == nullptr);
  const int M = a.M;

  // ---- set-up: barriers, TMEM, route compaction
  if (threadIdx.x == 0) {
    mbar_init(B.q_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&B.k_full[s], 1);
      mbar_init(&B.v_full[s], 1);
      mbar_init(&B.kv_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&B.s_full[b], 1);
      mbar_init(&B.s_free[b], 128);
    }
    mbar_init(B.p_full, 128);
    mbar_init(B.o_done, 1);
    mbar_init(B.mma_done, 1);
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
  const int n = *s_nvalid;
  const uint32_t tmem = *s_tmem;

  if (warp == 0) {
    // ================= TMA producer =================
    if (lane == 0 && n > 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      mbar_arrive_expect_tx(B.q_full, kTileBytes);
      tma_load_3d(sQ, &tmQ, B.q_full, 0, i * BM, h);
      tma_load_3d(sQ + kHalfBytes, &tmQ, B.q_full, 64, i * BM, h);
      int issued = 0;
      for (int j = 0; j < n; ++j) {
        const int s = j % NS;
        const uint32_t it = j / NS;
        if (!mbar_wait(&B.kv_empty[s], (it & 1) ^ 1, s_abort)) break;
        const int tile = dense ? j : tiles[j];
        mbar_arrive_expect_tx(&B.k_full[s], kTileBytes);
        tma_load_3d(sK + s * kTileBytes, &tmK, &B.k_full[s], 0, tile * BN, h);
        tma_load_3d(sK + s * kTileBytes + kHalfBytes, &tmK, &B.k_full[s], 64, tile * BN, h);
        mbar_arrive_expect_tx(&B.v_full[s], kTileBytes);
        tma_load_3d(sV + s * kTileBytes, &tmV, &B.v_full[s], 0, tile * BN, h);
        tma_load_3d(sV + s * kTileBytes + kHalfBytes, &tmV, &B.v_full[s], 64, tile * BN, h);
        issued = j + 1;
      }
      if (*s_abort) {
        // let the copies already in flight land before the CTA goes away
        // (each wait is bounded by the same time limit)
        volatile int never = 0;
        mbar_wait(B.q_full, 0, &never);
        for (int j = issued - NS < 0 ? 0 : issued - NS; j < issued; ++j) {
          const int s = j % NS;
          const uint32_t it = j / NS;
          never = 0;
          mbar_wait(&B.k_full[s], it & 1, &never);
          never = 0;
          mbar_wait(&B.v_full[s], it & 1, &never);
        }
      }
    }
  } else if (warp == 1) {
    // ================= MMA issuer =================
    if (lane == 0 && n > 0) {
      constexpr uint32_t idS = idesc_bf16_f32(BM, BN, false);
      constexpr uint32_t idPV = idesc_bf16_f32(BM, D, true);
      const uint32_t qa = smem_u32(sQ), pa = smem_u32(sP);
      bool ok = mbar_wait(B.q_full, 0, s_abort);
      tc_fence_after();
      auto issue_s = [&](int j) -> bool {
        const int s = j % NS, b = j & 1;
        if (!mbar_wait(&B.k_full[s], (j / NS) & 1, s_abort)) return false;
        if (!mbar_wait(&B.s_free[b], ((j >> 1) & 1) ^ 1, s_abort)) return false;
        tc_fence_after();
        const uint32_t ka = smem_u32(sK + s * kTileBytes);
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          mma_bf16_ss(tmem + b * BN, kmajor_desc(qa, k), kmajor_desc(ka, k), idS, k > 0);
        tc_commit(&B.s_full[b]);
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int j = 0; ok && j < n; ++j) {
        if (j + 1 < n && !issue_s(j + 1)) break;
        const int s = j % NS;
        if (!mbar_wait(B.p_full, j & 1, s_abort)) break;
        if (!mbar_wait(&B.v_full[s], (j / NS) & 1, s_abort)) break;
        tc_fence_after();
        const uint32_t va = smem_u32(sV + s * kTileBytes);
#pragma unroll
        for (int k = 0; k < BN / 16; ++k)
          mma_bf16_ss(tmem + kColO, kmajor_desc(pa, k), vmn_desc(va, k), idPV, (j > 0 || k > 0));
        tc_commit(&B.kv_empty[s]);
        tc_commit(B.o_done);
      }
      // all issued MMAs must be complete before TMEM is released
      tc_commit(B.mma_done);
      volatile int never = 0;
      mbar_wait(B.mma_done, 0, &never);
    }
  } else {
    // ================= softmax / epilogue (warps 2..5) =================
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // query row within the tile = TMEM lane
    const uint32_t trow = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const int b = j & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&B.s_full[b], (j >> 1) & 1, s_abort))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sv[128];
#pragma unroll
      for (int c = 0; c < 4; ++c)
        tmem_ld32(trow + b * BN + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[c * 32]));
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&B.s_free[b]);
      float mx = -INFINITY;
#pragma unroll
      for (int k = 0; k < 128; ++k) mx = fmaxf(mx, __uint_as_float(sv[k]));
      const float m_new = fmaxf(m, mx * a.scale_log2);
      uint32_t pk[64];
      float sum = 0.f;
#pragma unroll
      for (int k = 0; k < 64; ++k) {
        const float p0 = fast_exp2(fmaf(__uint_as_float(sv[2 * k]), a.scale_log2, -m_new));
        const float p1 = fast_exp2(fmaf(__uint_as_float(sv[2 * k + 1]), a.scale_log2, -m_new));
        sum += p0 + p1;
        pk[k] = pack_bf16x2(p0, p1);
      }
      const float alpha = fast_exp2(m - m_new);  // 0 on the first tile
      if (j > 0) {
        if (!__all_sync(0xffffffffu, mbar_wait(B.o_done, (j - 1) & 1, s_abort))) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (__any_sync(0xffffffffu, m_new > m)) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t ov[32];
            tmem_ld32(trow + kColO + c * 32, ov);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 32; ++k) ov[k] = __float_as_uint(__uint_as_float(ov[k]) * alpha);
            tmem_st32(trow + kColO + c * 32, ov);
          }
          tmem_wait_st();
        }
      }
      l = l * alpha + sum;
      m = m_new;
      // P row -> shared memory, K-major 128-byte swizzle (same layout TMA
      // gives Q and K): 16-byte chunk c of row r lands at chunk c ^ (r & 7).
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        uint8_t *dst = sP + (c >> 3) * kHalfBytes + r * 128 + (((c & 7) ^ (r & 7)) << 4);
        *reinterpret_cast<uint4 *>(dst) = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(B.p_full);
    }
    // epilogue
    uint16_t *orow = a.O + ((size_t)row * BM + r) * D;
    bool have = ok && n > 0;
    if (have) have = mbar_wait(B.o_done, (n - 1) & 1, s_abort);
    // tcgen05.ld is warp-collective: decide once for the whole warp
    const bool good = __all_sync(0xffffffffu, have && !*s_abort);
    tc_fence_after();
    const float inv = good ? 1.0f / l : 0.f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t ov[32];
      if (good) {
        tmem_ld32(trow + kColO + c * 32, ov);
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
        *reinterpret_cast<uint4 *>(orow + c * 32 + q * 8) = v;
      }
    }
    if (a.lse) a.lse[(size_t)row * BM + r] = good ? (m + __log2f(l)) * 0.69314718055994531f : -INFINITY;
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
                        const int32_t *route_ids, const int32_t *route_len, int R_max, int H,
                        int N, int M, float softmax_scale, uint16_t *O, float *lse,
                        int32_t *dev_status, cudaStream_t stream, bool *map_failed) {
  *map_failed = false;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, Q, N * BM, H) || !make_map(&mk, K, M * BN, H) ||
      !make_map(&mv, V, M * BN, H)) {
    *map_failed = true;
    return cudaErrorInvalidValue;
  }
  AttnArgs a;
  a.route_ids = route_ids;
  a.route_len = route_len;
  a.R_max = R_max;
  a.N = N;
  a.M = M;
  a.scale_log2 = softmax_scale * 1.4426950408889634f;
  a.O = O;
  a.lse = lse;
  a.dev_status = dev_status;
  cudaError_t e = cudaFuncSetAttribute(attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  attn_kernel<<<H * N, kThreads, kSmemBytes, stream>>>(mq, mk, mv, a);
  return cudaGetLastError();
}

}  // namespace velox

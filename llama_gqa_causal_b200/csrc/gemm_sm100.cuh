// bf16 GEMM on the 5th-generation tensor cores for the projections around
// attention ("[HuggingFace Transformers] LlamaAttention source walkthrough",
// section 2 forward() step 1: q/k/v = x W_q^T, x W_k^T, x W_v^T, and step 7:
// o_proj; "Llama2 Transformer architecture and optimisation practice",
// section 2.1: RoPE applies to Q and K after projection):
//   Y[M, N] = X[M, K] . W[N, K]^T
// with W in the nn.Linear layout, so both operands are K-major in shared
// memory.  Two epilogues:
//   plain   Y stored as bf16 [M, N]
//   qkv     the columns are the heads of [W_q; W_k; W_v]: each 128-row tile's
//           head is rotated with RoPE (q and k heads, cos/sin of the row's
//           token) and stored to q [M, H, D], k [M, Hkv, D] or v [M, Hkv, D]
//           -- the layouts the attention entry points take, already rotated.
//
// Tile 128 x 256 (one M = 128, N = 256 tcgen05 MMA per 16-wide k-step: the
// operands are 4 KB of X and 8 KB of W per 128 cycles, inside what the tensor
// core reads from shared memory per cycle), K in blocks of 64 (one 128-byte
// swizzle row) through a 4-stage TMA ring.
// Persistent: one CTA per SM walks tiles blockIdx.x, + gridDim.x, ...  The
// accumulator is double-buffered in TMEM (2 x 256 columns, all of it), so the
// epilogue of one tile runs while the MMAs of the next fill the other buffer.
// Warps: 0 TMA producer, 1 TMEM allocator + MMA issuer, 2-5 epilogue (one
// output row per thread; warp w reaches TMEM lanes of quarter w % 4).
#pragma once
#include "common.cuh"

namespace la {
namespace gm {
constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;
constexpr int STAGES = 4;
constexpr int THREADS = 192;
constexpr uint32_t A_BYTES = BM * BK * 2;  // 16 KB
constexpr uint32_t B_BYTES = BN * BK * 2;  // 32 KB
// Tiles are taken in groups of GROUP_M row tiles that sweep every column tile
// before the next group starts: a group's rows of X (16 x 128 rows) stay in L2
// while W streams past, so X is read from DRAM about once and W once per group.
constexpr int GROUP_M = 16;
}  // namespace gm

struct GemmParams {
  int M, N, K;
  __nv_bfloat16* y;                  // plain: [M, N]
  __nv_bfloat16* q;                  // qkv: [M, H, D]
  __nv_bfloat16* k;                  // qkv: [M, Hkv, D]
  __nv_bfloat16* v;                  // qkv: [M, Hkv, D]
  const float* cos;                  // qkv: [M, D] of each row's token, or null (no RoPE)
  const float* sin;
  int H, Hkv;
};

struct GmSmem {
  alignas(1024) __nv_bfloat16 a[gm::STAGES][gm::BM * gm::BK];
  alignas(1024) __nv_bfloat16 b[gm::STAGES][gm::BN * gm::BK];
  uint64_t full[gm::STAGES], empty[gm::STAGES];
  uint64_t acc_full[2];   // accumulator buffer holds a finished tile (MMA commit)
  uint64_t acc_empty[2];  // its epilogue has read it (one arrive per epilogue warp)
  uint64_t mma_done;      // every MMA this CTA issued has completed
  uint32_t tmem_base;
};

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* m, uint64_t* bar, int c0,
                                            int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}

// QKV (true): the rotating epilogue for heads of D columns; plain (false): D unused.
template <bool QKV, int D>
__global__ void __launch_bounds__(gm::THREADS, 1)
    gemm_bf16_kernel(const __grid_constant__ CUtensorMap tm_a,
                     const __grid_constant__ CUtensorMap tm_b, GemmParams p) {
  using namespace gm;
  constexpr uint32_t TMEM_COLS = 2 * BN;
  constexpr uint32_t IDESC = idesc_bf16(BM, BN, false);
  extern __shared__ uint8_t smem_raw[];
  GmSmem& s = *reinterpret_cast<GmSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_m = (p.M + BM - 1) / BM, n_n = (p.N + BN - 1) / BN;
  const int n_tiles = n_m * n_n;
  const int nk = (p.K + BK - 1) / BK;
  // tile index -> (first row, first column)
  auto tile_origin = [&](int tile, int& m0, int& n0) {
    const int group = tile / (GROUP_M * n_n);
    const int first_m = group * GROUP_M;
    const int gsize = min(GROUP_M, n_m - first_m);
    const int local = tile - group * GROUP_M * n_n;
    m0 = (first_m + local % gsize) * BM;
    n0 = (local / gsize) * BN;
  };

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.acc_full[i], 1);
      mbar_init(&s.acc_empty[i], 4);
    }
    mbar_init(&s.mma_done, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&s.tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (elect_one()) {
      tma_prefetch_desc(&tm_a);
      tma_prefetch_desc(&tm_b);
    }
    __syncwarp();
    int it = 0;  // k-blocks issued by this CTA, over all its tiles
    bool ok = true;
    for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
      int m0, n0;
      tile_origin(tile, m0, n0);
      for (int kb = 0; kb < nk; ++kb, ++it) {
        const int st = it % STAGES;
        if (it >= STAGES && !mbar_wait(&s.empty[st], ((it / STAGES) - 1) & 1)) {
          ok = false;
          break;
        }
        if (elect_one()) {
          mbar_arrive_expect_tx(&s.full[st], A_BYTES + B_BYTES);
          tma_load_2d(&s.a[st][0], &tm_a, &s.full[st], kb * BK, m0);
          tma_load_2d(&s.b[st][0], &tm_b, &s.full[st], kb * BK, n0);
        }
        __syncwarp();
      }
    }
    // leave no copy in flight
    for (int i = max(0, it - STAGES); i < it; ++i)
      if (!mbar_wait(&s.full[i % STAGES], (i / STAGES) & 1)) break;
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const uint64_t a_desc0 = sw128_desc(smem_u32(&s.a[0][0]), 16, 1024);
    const uint64_t b_desc0 = sw128_desc(smem_u32(&s.b[0][0]), 16, 1024);
    bool ok = true;
    int it = 0;  // k-blocks consumed, over all tiles
    int i = 0;   // tiles of this CTA
    for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x, ++i) {
      const int acc = i & 1;
      // the epilogue has read this buffer's previous tile (i - 2)
      if (i >= 2 && !mbar_wait(&s.acc_empty[acc], ((i >> 1) - 1) & 1)) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem + static_cast<uint32_t>(acc * BN);
      for (int kb = 0; kb < nk; ++kb, ++it) {
        const int st = it % STAGES;
        ok = mbar_wait(&s.full[st], (it / STAGES) & 1);
        if (!ok) break;
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = a_desc0 + ((static_cast<uint32_t>(st) * A_BYTES + kk * 32) >> 4);
            const uint64_t bd = b_desc0 + ((static_cast<uint32_t>(st) * B_BYTES + kk * 32) >> 4);
            mma_ss(d_tmem, ad, bd, IDESC, (kb > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(&s.empty[st]);
        }
        __syncwarp();
      }
      if (!ok) break;
      if (elect_one()) tc_commit(&s.acc_full[acc]);  // the tile's MMAs have completed when it fires
      __syncwarp();
    }
    // no MMA may still run when the TMEM is released
    if (elect_one()) tc_commit(&s.mma_done);
    __syncwarp();
    mbar_wait(&s.mma_done, 0);
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    int i = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++i) {
      const int acc = i & 1;
      int m0, n0;
      tile_origin(tile, m0, n0);
      const int m = m0 + r;  // output row (token)
      const bool row_ok = m < p.M;
      if (!mbar_wait(&s.acc_full[acc], (i >> 1) & 1)) break;
      tc_fence_after();
      const uint32_t t_acc = tmem + static_cast<uint32_t>(acc * BN) +
                             (static_cast<uint32_t>(quarter * 32) << 16);
      if constexpr (!QKV) {
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t acc_r[32];
          tmem_ld32(t_acc + c * 32, acc_r);
          tmem_ld_wait(acc_r);
          const int n = n0 + c * 32;
          if (row_ok && n < p.N) {
            __nv_bfloat16* dst = p.y + static_cast<size_t>(m) * p.N + n;
#pragma unroll
            for (int e = 0; e < 32; e += 8) {
              if (n + e + 8 <= p.N) {
                uint4 w;
                w.x = pack_bf16x2(__uint_as_float(acc_r[e]), __uint_as_float(acc_r[e + 1]));
                w.y = pack_bf16x2(__uint_as_float(acc_r[e + 2]), __uint_as_float(acc_r[e + 3]));
                w.z = pack_bf16x2(__uint_as_float(acc_r[e + 4]), __uint_as_float(acc_r[e + 5]));
                w.w = pack_bf16x2(__uint_as_float(acc_r[e + 6]), __uint_as_float(acc_r[e + 7]));
                *reinterpret_cast<uint4*>(dst + e) = w;
              }
            }
          }
        }
      } else {
        const int mt = row_ok ? m : p.M - 1;  // table row (any valid one for rows past M)
        const float* crow = p.cos ? p.cos + static_cast<size_t>(mt) * D : nullptr;
        const float* srow = p.sin ? p.sin + static_cast<size_t>(mt) * D : nullptr;
#pragma unroll 1
        for (int hl = 0; hl < BN / D; ++hl) {
          const int nh = n0 + hl * D;  // first column of this head
          // which projection and head the columns belong to
          __nv_bfloat16* dst = nullptr;
          bool rotate = false;
          if (nh < p.H * D) {
            dst = p.q + (static_cast<size_t>(m) * p.H + nh / D) * D;
            rotate = crow != nullptr;
          } else if (nh < (p.H + p.Hkv) * D) {
            dst = p.k + (static_cast<size_t>(m) * p.Hkv + (nh - p.H * D) / D) * D;
            rotate = crow != nullptr;
          } else {
            dst = p.v + (static_cast<size_t>(m) * p.Hkv + (nh - (p.H + p.Hkv) * D) / D) * D;
          }
          const bool store = row_ok && nh < p.N;
#pragma unroll 1
          for (int j = 0; j < D / 64; ++j) {
            // columns d in [32j, 32j + 32) and their rotation partners d + D/2
            uint32_t x1[32], x2[32];
            tmem_ld32(t_acc + hl * D + 32 * j, x1);
            tmem_ld32(t_acc + hl * D + D / 2 + 32 * j, x2);
            tmem_ld_wait(x1);
            tmem_ld_wait(x2);
#pragma unroll
            for (int e = 0; e < 32; e += 8) {
              float y1[8], y2[8];
#pragma unroll
              for (int u = 0; u < 8; ++u) {
                y1[u] = __uint_as_float(x1[e + u]);
                y2[u] = __uint_as_float(x2[e + u]);
              }
              if (rotate) {
                const int d = 32 * j + e;
                const float4 c1a = *reinterpret_cast<const float4*>(crow + d);
                const float4 c1b = *reinterpret_cast<const float4*>(crow + d + 4);
                const float4 c2a = *reinterpret_cast<const float4*>(crow + D / 2 + d);
                const float4 c2b = *reinterpret_cast<const float4*>(crow + D / 2 + d + 4);
                const float4 s1a = *reinterpret_cast<const float4*>(srow + d);
                const float4 s1b = *reinterpret_cast<const float4*>(srow + d + 4);
                const float4 s2a = *reinterpret_cast<const float4*>(srow + D / 2 + d);
                const float4 s2b = *reinterpret_cast<const float4*>(srow + D / 2 + d + 4);
                const float c1[8] = {c1a.x, c1a.y, c1a.z, c1a.w, c1b.x, c1b.y, c1b.z, c1b.w};
                const float c2[8] = {c2a.x, c2a.y, c2a.z, c2a.w, c2b.x, c2b.y, c2b.z, c2b.w};
                const float s1[8] = {s1a.x, s1a.y, s1a.z, s1a.w, s1b.x, s1b.y, s1b.z, s1b.w};
                const float s2[8] = {s2a.x, s2a.y, s2a.z, s2a.w, s2b.x, s2b.y, s2b.z, s2b.w};
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                  const float a = y1[u], z = y2[u];
                  y1[u] = fmaf(a, c1[u], -z * s1[u]);  // x cos + rotate_half(x) sin, first half
                  y2[u] = fmaf(z, c2[u], a * s2[u]);   // second half
                }
              }
              if (store) {
                uint4 w1, w2;
                w1.x = pack_bf16x2(y1[0], y1[1]);
                w1.y = pack_bf16x2(y1[2], y1[3]);
                w1.z = pack_bf16x2(y1[4], y1[5]);
                w1.w = pack_bf16x2(y1[6], y1[7]);
                w2.x = pack_bf16x2(y2[0], y2[1]);
                w2.y = pack_bf16x2(y2[2], y2[3]);
                w2.z = pack_bf16x2(y2[4], y2[5]);
                w2.w = pack_bf16x2(y2[6], y2[7]);
                *reinterpret_cast<uint4*>(dst + 32 * j + e) = w1;
                *reinterpret_cast<uint4*>(dst + D / 2 + 32 * j + e) = w2;
              }
            }
          }
        }
      }
      // every tcgen05.ld of this buffer has completed (waited above): hand it
      // back to the MMA warp for tile i + 2
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.acc_empty[acc]);
    }
  }

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace la

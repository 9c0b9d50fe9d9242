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
  uint64_t acc_full;
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
  constexpr uint32_t TMEM_COLS = BN;
  constexpr uint32_t IDESC = idesc_bf16(BM, BN, false);
  extern __shared__ uint8_t smem_raw[];
  GmSmem& s = *reinterpret_cast<GmSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_m = (p.M + BM - 1) / BM, n_n = (p.N + BN - 1) / BN;
  const int group = blockIdx.x / (GROUP_M * n_n);
  const int first_m = group * GROUP_M;
  const int gsize = min(GROUP_M, n_m - first_m);
  const int local = blockIdx.x - group * GROUP_M * n_n;
  const int m0 = (first_m + local % gsize) * BM, n0 = (local / gsize) * BN;
  const int nk = (p.K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    mbar_init(&s.acc_full, 1);
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
    int issued = 0;
    for (int kb = 0; kb < nk; ++kb) {
      const int st = kb % STAGES;
      if (kb >= STAGES && !mbar_wait(&s.empty[st], ((kb / STAGES) - 1) & 1)) break;
      if (elect_one()) {
        mbar_arrive_expect_tx(&s.full[st], A_BYTES + B_BYTES);
        tma_load_2d(&s.a[st][0], &tm_a, &s.full[st], kb * BK, m0);
        tma_load_2d(&s.b[st][0], &tm_b, &s.full[st], kb * BK, n0);
      }
      __syncwarp();
      issued = kb + 1;
    }
    // leave no copy in flight
    for (int kb = max(0, issued - STAGES); kb < issued; ++kb)
      if (!mbar_wait(&s.full[kb % STAGES], (kb / STAGES) & 1)) break;
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const uint64_t a_desc0 = sw128_desc(smem_u32(&s.a[0][0]), 16, 1024);
    const uint64_t b_desc0 = sw128_desc(smem_u32(&s.b[0][0]), 16, 1024);
    bool ok = true;
    for (int kb = 0; kb < nk && ok; ++kb) {
      const int st = kb % STAGES;
      ok = mbar_wait(&s.full[st], (kb / STAGES) & 1);
      if (!ok) break;
      tc_fence_after();
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          const uint64_t ad = a_desc0 + ((static_cast<uint32_t>(st) * A_BYTES + kk * 32) >> 4);
          const uint64_t bd = b_desc0 + ((static_cast<uint32_t>(st) * B_BYTES + kk * 32) >> 4);
          mma_ss(tmem, ad, bd, IDESC, (kb > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(&s.empty[st]);
      }
      __syncwarp();
    }
    if (elect_one()) tc_commit(&s.acc_full);  // every MMA above has completed when it fires
    __syncwarp();
    mbar_wait(&s.acc_full, 0);
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int m = m0 + r;  // output row (token)
    const bool row_ok = m < p.M;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    if (mbar_wait(&s.acc_full, 0)) {
      tc_fence_after();
      if constexpr (!QKV) {
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t acc[32];
          tmem_ld32(tmem + lane_off + c * 32, acc);
          tmem_ld_wait(acc);
          const int n = n0 + c * 32;
          if (row_ok && n < p.N) {
            __nv_bfloat16* dst = p.y + static_cast<size_t>(m) * p.N + n;
#pragma unroll
            for (int e = 0; e < 32; e += 8) {
              if (n + e + 8 <= p.N) {
                uint4 w;
                w.x = pack_bf16x2(__uint_as_float(acc[e]), __uint_as_float(acc[e + 1]));
                w.y = pack_bf16x2(__uint_as_float(acc[e + 2]), __uint_as_float(acc[e + 3]));
                w.z = pack_bf16x2(__uint_as_float(acc[e + 4]), __uint_as_float(acc[e + 5]));
                w.w = pack_bf16x2(__uint_as_float(acc[e + 6]), __uint_as_float(acc[e + 7]));
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
            tmem_ld32(tmem + lane_off + hl * D + 32 * j, x1);
            tmem_ld32(tmem + lane_off + hl * D + D / 2 + 32 * j, x2);
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

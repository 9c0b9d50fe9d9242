// bf16 split-KV decode: one query token per sequence against a KV cache
// ("LLaMA2 large language model architecture analysis", section "KV cache":
// the new token's single query row attends to every cached key; section
// "GQA": several query heads share each K/V head, so one read of a K/V row
// serves the whole group).
//
// Grid (split, kv_head x head_chunk, batch).  A CTA streams rows
// [split*C, min((split+1)*C, len)) of one K/V head through a ring of TMA
// stages (64 rows of K and V each, 128-byte swizzle) and computes, for up to
// 8 query heads of the group at once, the partial softmax state (running max
// m, sum l, un-normalised output o) over those rows.  Four consumer warps take
// 16 rows of each stage:
//   S^T[16 keys x 8 heads]  = K[16 x D] . Q'^T[D x 8]     (mma m16n8k16, K from
//                                                          ldmatrix, Q' in regs)
//   O^T[D x 8 heads]       += V^T[D x 16] . P^T[16 x 8]    (V^T by ldmatrix.trans,
//                                                          P^T by movmatrix)
// so no tensor work is spent on padding when the group has 8 heads.  The
// partial states of the four warps are merged in shared memory and written to
// the workspace; decode_combine_kernel merges the splits with the
// log-sum-exp identity and writes bf16 output.
#pragma once
#include "common.cuh"

namespace la {
namespace dec {
constexpr int TR = 64;      // cache rows per stage
constexpr int NCW = 4;      // consumer warps (16 rows of a stage each)
constexpr int NSTAGE = 3;   // ring depth
constexpr int THREADS = (NCW + 1) * 32;
}  // namespace dec

struct DecodeParams {
  const __nv_bfloat16* q;  // [b, H, D] un-rotated
  const float* cos;        // [b, D] or null
  const float* sin;
  const int* lens;         // [b]
  float* ws_o;             // [b, H, n_splits, D]
  float* ws_ml;            // [b, H, n_splits, 2]
  int bsz, H, Hkv, L, group, hchunks, split_rows, n_splits;
  float scale_log2;        // scale * log2(e)
};

template <int D>
struct DecSmem {
  alignas(1024) __nv_bfloat16 k[dec::NSTAGE][dec::TR * D];
  alignas(1024) __nv_bfloat16 v[dec::NSTAGE][dec::TR * D];
  uint64_t full[dec::NSTAGE];
  uint64_t empty[dec::NSTAGE];
  float red_m[dec::NCW][8];
  float red_l[dec::NCW][8];
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr)
               : "memory");
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr)
               : "memory");
}
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int D>
__global__ void __launch_bounds__(dec::THREADS) decode_bf16_kernel(
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
    DecodeParams p) {
  using namespace dec;
  constexpr int KSTEPS = D / 16;  // k-steps of the QK^T product, m-tiles of PV
  constexpr int CB = D / 64;      // 64-column swizzle blocks per row
  constexpr uint32_t STAGE_BLOCK_BYTES = TR * 64 * 2;  // one [64 rows x 64 cols] block
  extern __shared__ uint8_t smem_raw[];
  DecSmem<D>& s = *reinterpret_cast<DecSmem<D>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x;
  const int kvh = blockIdx.y / p.hchunks, hc = blockIdx.y - kvh * p.hchunks;
  const int b = blockIdx.z;
  int len = p.lens[b];
  len = len < 0 ? 0 : (len > p.L ? p.L : len);
  const int start = split * p.split_rows;
  if (start >= len) return;  // uniform across the block, before any barrier
  const int rows = min(p.split_rows, len - start);
  const int nT = (rows + TR - 1) / TR;
  const int bh = b * p.Hkv + kvh;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NSTAGE; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], NCW);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == NCW) {  // ---------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int issued = 0;
      for (int it = 0; it < nT; ++it) {
        const int st = it % NSTAGE;
        if (it >= NSTAGE && !mbar_wait(&s.empty[st], ((it / NSTAGE) - 1) & 1)) break;
        mbar_arrive_expect_tx(&s.full[st], 2u * TR * D * 2u);
#pragma unroll
        for (int cb = 0; cb < CB; ++cb) {
          tma_load_3d(&s.k[st][cb * TR * 64], &tm_k, &s.full[st], cb * 64, start + it * TR, bh);
          tma_load_3d(&s.v[st][cb * TR * 64], &tm_v, &s.full[st], cb * 64, start + it * TR, bh);
        }
        issued = it + 1;
      }
      // never leave with copies in flight: wait for every issued stage to land
      for (int it = max(0, issued - NSTAGE); it < issued; ++it)
        if (!mbar_wait(&s.full[it % NSTAGE], (it / NSTAGE) & 1)) break;
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  const int g = lane >> 2, t = lane & 3;
  const int hq = hc * 8 + g;  // query head within the group held by this lane's B columns
  const bool hvalid = hq < p.group;
  // Q' fragments: lane holds head hq, dims kk*16 + 2t + {0, 1, 8, 9}.  The
  // rotation partner of dim d is d +- D/2, i.e. k-step kk +- D/32, same lane.
  uint32_t qf[KSTEPS][2];
  {
    float qx[KSTEPS][4];
    const __nv_bfloat16* qr = p.q + (static_cast<size_t>(b) * p.H + kvh * p.group + hq) * D;
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int d = kk * 16 + 2 * t + (j < 2 ? j : j + 6);
        qx[kk][j] = hvalid ? __bfloat162float(qr[d]) : 0.f;
      }
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk) {
      float y[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        y[j] = qx[kk][j];
        if (p.cos != nullptr) {
          const int d = kk * 16 + 2 * t + (j < 2 ? j : j + 6);
          const float c = p.cos[static_cast<size_t>(b) * D + d];
          const float sn = p.sin[static_cast<size_t>(b) * D + d];
          const float rot = (kk < KSTEPS / 2) ? -qx[kk + KSTEPS / 2][j] : qx[kk - KSTEPS / 2][j];
          y[j] = fmaf(qx[kk][j], c, rot * sn);
        }
      }
      qf[kk][0] = pack_bf16x2(y[0], y[1]);
      qf[kk][1] = pack_bf16x2(y[2], y[3]);
    }
  }

  float m_run[2] = {-INFINITY, -INFINITY};
  float l_run[2] = {0.f, 0.f};
  float o[KSTEPS][4];
#pragma unroll
  for (int mt = 0; mt < KSTEPS; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;

  const int mat = lane >> 3, r8 = lane & 7;
  bool ok = true;
  for (int it = 0; it < nT; ++it) {
    const int st = it % NSTAGE;
    if (!mbar_wait(&s.full[st], (it / NSTAGE) & 1)) { ok = false; break; }
    const int key0 = start + it * TR + warp * 16;
    const int nvalid = min(16, len - key0);
    const uint32_t kbase = smem_u32(&s.k[st][0]);
    const uint32_t vbase = smem_u32(&s.v[st][0]);
    if (nvalid > 0) {
      if (nvalid < 16) {
        // cache rows at or past the length may hold anything (NaN): zero this
        // warp's V rows there so that 0-weight keys add exactly 0
        uint8_t* vb = reinterpret_cast<uint8_t*>(&s.v[st][0]);
        for (int idx = lane; idx < (16 - nvalid) * CB * 8; idx += 32) {
          const int rr = warp * 16 + nvalid + idx / (CB * 8);
          const int rem = idx % (CB * 8);
          *reinterpret_cast<uint4*>(vb + (rem / 8) * STAGE_BLOCK_BYTES +
                                    sw128_offset(rr, rem % 8)) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
        __syncwarp();
      }
      // ---- S^T = K Q'^T over this warp's 16 keys
      float sc[4] = {0.f, 0.f, 0.f, 0.f};
      const int krow = warp * 16 + (mat & 1) * 8 + r8;
#pragma unroll
      for (int kk = 0; kk < KSTEPS; ++kk) {
        const int col = kk * 16 + (mat >> 1) * 8;
        uint32_t a0, a1, a2, a3;
        ldsm_x4(kbase + (col / 64) * STAGE_BLOCK_BYTES + sw128_offset(krow, (col % 64) / 8), a0,
                a1, a2, a3);
        mma_bf16_16816(sc, a0, a1, a2, a3, qf[kk][0], qf[kk][1]);
      }
      // sc[0]=(key g, head 2t) sc[1]=(key g, head 2t+1) sc[2]=(key g+8, 2t) sc[3]=(key g+8, 2t+1)
      const bool v0 = g < nvalid, v1 = g + 8 < nvalid;
      float x[4];
      x[0] = v0 ? sc[0] * p.scale_log2 : -INFINITY;
      x[1] = v0 ? sc[1] * p.scale_log2 : -INFINITY;
      x[2] = v1 ? sc[2] * p.scale_log2 : -INFINITY;
      x[3] = v1 ? sc[3] * p.scale_log2 : -INFINITY;
      float alpha[2], pr[4];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float mx = fmaxf(x[h], x[h + 2]);
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        const float m_new = fmaxf(m_run[h], mx);  // finite: key0 < len is valid
        alpha[h] = (m_run[h] == -INFINITY) ? 0.f : ex2_approx(m_run[h] - m_new);
        pr[h] = ex2_approx(x[h] - m_new);
        pr[h + 2] = ex2_approx(x[h + 2] - m_new);
        l_run[h] = fmaf(l_run[h], alpha[h], pr[h] + pr[h + 2]);
        m_run[h] = m_new;
      }
#pragma unroll
      for (int mt = 0; mt < KSTEPS; ++mt) {
        o[mt][0] *= alpha[0];
        o[mt][1] *= alpha[1];
        o[mt][2] *= alpha[0];
        o[mt][3] *= alpha[1];
      }
      // P^T fragments for the PV product (keys = k dim, heads = n dim)
      const uint32_t pb0 = movmatrix_t(pack_bf16x2(pr[0], pr[1]));
      const uint32_t pb1 = movmatrix_t(pack_bf16x2(pr[2], pr[3]));
      // ---- O^T += V^T P^T
      const int vrow = warp * 16 + (mat >> 1) * 8 + r8;
#pragma unroll
      for (int mt = 0; mt < KSTEPS; ++mt) {
        const int col = mt * 16 + (mat & 1) * 8;
        uint32_t a0, a1, a2, a3;
        ldsm_x4_t(vbase + (col / 64) * STAGE_BLOCK_BYTES + sw128_offset(vrow, (col % 64) / 8),
                  a0, a1, a2, a3);
        mma_bf16_16816(o[mt], a0, a1, a2, a3, pb0, pb1);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.empty[st]);
  }

  // ---- merge the four warps' partial states (stage memory reused as scratch)
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 4);
    l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 8);
    l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 16);
  }
  named_bar_sync(1, NCW * 32);  // every warp is done reading the stages
  if (!ok) return;               // a wait ran out: leave without writing
  float* red_o = reinterpret_cast<float*>(&s.k[0][0]);  // [NCW][8][D]
  if (g == 0) {
    s.red_m[warp][2 * t] = m_run[0];
    s.red_m[warp][2 * t + 1] = m_run[1];
    s.red_l[warp][2 * t] = l_run[0];
    s.red_l[warp][2 * t + 1] = l_run[1];
  }
#pragma unroll
  for (int mt = 0; mt < KSTEPS; ++mt) {
    red_o[(warp * 8 + 2 * t) * D + mt * 16 + g] = o[mt][0];
    red_o[(warp * 8 + 2 * t + 1) * D + mt * 16 + g] = o[mt][1];
    red_o[(warp * 8 + 2 * t) * D + mt * 16 + g + 8] = o[mt][2];
    red_o[(warp * 8 + 2 * t + 1) * D + mt * 16 + g + 8] = o[mt][3];
  }
  named_bar_sync(1, NCW * 32);
  {
    constexpr int PER = D / 16;  // dims per thread: 128 threads cover 8 heads x D
    const int tid = threadIdx.x;
    const int hh = tid >> 4;
    const int d0 = (tid & 15) * PER;
    const int hq2 = hc * 8 + hh;
    if (hq2 < p.group) {
      float mstar = -INFINITY;
#pragma unroll
      for (int w = 0; w < NCW; ++w) mstar = fmaxf(mstar, s.red_m[w][hh]);
      float f[NCW], lsum = 0.f;
#pragma unroll
      for (int w = 0; w < NCW; ++w) {
        const float mw = s.red_m[w][hh];
        f[w] = (mw == -INFINITY) ? 0.f : ex2_approx(mw - mstar);
        lsum = fmaf(f[w], s.red_l[w][hh], lsum);
      }
      const int head = kvh * p.group + hq2;
      const size_t slot = (static_cast<size_t>(b) * p.H + head) * p.n_splits + split;
      float* dst = p.ws_o + slot * D + d0;
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < NCW; ++w) acc = fmaf(f[w], red_o[(w * 8 + hh) * D + d0 + i], acc);
        dst[i] = acc;
      }
      if ((tid & 15) == 0) {
        p.ws_ml[slot * 2] = mstar;
        p.ws_ml[slot * 2 + 1] = lsum;
      }
    }
  }
}

// Merge the per-split partial states of one (b, head):
//   m* = max_s m_s,  l = sum_s l_s 2^(m_s - m*),  o = sum_s o_s 2^(m_s - m*) / l.
template <int D>
__global__ void __launch_bounds__(D) decode_combine_kernel(const float* __restrict__ ws_o,
                                                           const float* __restrict__ ws_ml,
                                                           const int* __restrict__ lens,
                                                           __nv_bfloat16* __restrict__ out,
                                                           int H, int L, int split_rows,
                                                           int n_splits) {
  const int h = blockIdx.x, b = blockIdx.y, d = threadIdx.x;
  int len = lens[b];
  len = len < 0 ? 0 : (len > L ? L : len);
  const int n = (len + split_rows - 1) / split_rows;
  const size_t slot0 = (static_cast<size_t>(b) * H + h) * n_splits;
  float mstar = -INFINITY;
  for (int s = 0; s < n; ++s) mstar = fmaxf(mstar, ws_ml[(slot0 + s) * 2]);
  float lsum = 0.f, acc = 0.f;
  for (int s = 0; s < n; ++s) {
    const float f = ex2_approx(ws_ml[(slot0 + s) * 2] - mstar);
    lsum = fmaf(f, ws_ml[(slot0 + s) * 2 + 1], lsum);
    acc = fmaf(f, ws_o[(slot0 + s) * D + d], acc);
  }
  const float r = (lsum > 0.f) ? acc / lsum : 0.f;
  out[(static_cast<size_t>(b) * H + h) * D + d] = __float2bfloat16_rn(r);
}

}  // namespace la

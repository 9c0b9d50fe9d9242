// fp32 attention on CUDA cores (FFMA only, no TF32): prefill and decode.
//
// Computes, per query row, softmax(scale * q'.k'_j + mask_j) . v_j in fp32
// ("[HuggingFace Transformers] LlamaAttention source walkthrough", section
// 1.2 steps 2-4, section 2 steps 3-5.3), with q' and k' rotated by RoPE in
// the kernel and the K/V head chosen by the repeat_kv map h / group.
//
// Block = 128 threads = 32 query rows x 4 lanes; lane e of a row owns the
// dims d = e + 4m.  K/V are staged 32 keys at a time in shared memory (K
// rotated on the way in).  The online softmax keeps a running max and sum per
// row and rescales the accumulator once per key tile (exact arithmetic; expf).
//
// Prefill: rows = 32 consecutive positions of one query head; grid
//   (ceil(S/32), H, bsz).  Decode: rows = the query heads of one K/V group
//   (chunks of 32); grid (ceil(group/32), Hkv, bsz); keys = the first
//   cache_lens[b] cache rows (already rotated), no causal mask.
#pragma once
#include "common.cuh"

namespace la {

struct Fp32Params {
  const float* q;
  const float* k;
  const float* v;
  const float* cos;   // prefill [b, S, D] ; decode [b, D] ; or null
  const float* sin;
  const float* mask;  // prefill only: [b, 1, S, S] or null
  const int* lens;    // decode only
  float* out;
  int bsz, H, Hkv, S, L, group;
  int decode, causal;
  float scale;
};

template <int D>
__global__ void __launch_bounds__(128) attn_fp32_kernel(Fp32Params p) {
  constexpr int KT = 32;       // keys per tile
  constexpr int DL = D / 4;    // dims per lane
  __shared__ float ks[KT][D + 4];
  __shared__ float vs[KT][D + 4];

  const int tid = threadIdx.x;
  const int row = tid >> 2;   // 0..31
  const int e = tid & 3;      // lane within the row
  const int b = blockIdx.z;

  int head, kvh, qi;          // query head, K/V head, query position (prefill)
  bool active;
  int n_keys;
  if (!p.decode) {
    head = blockIdx.y;
    kvh = head / p.group;
    qi = blockIdx.x * 32 + row;
    active = qi < p.S;
    n_keys = p.causal ? min(p.S, blockIdx.x * 32 + 32) : p.S;
  } else {
    kvh = blockIdx.y;
    const int hh = blockIdx.x * 32 + row;
    head = kvh * p.group + hh;
    qi = 0;
    active = hh < p.group;
    int len = p.lens[b];
    len = len < 0 ? 0 : (len > p.L ? p.L : len);
    n_keys = len;
  }

  // ---- load + rotate this row's query slice
  float qv[DL], acc[DL];
  {
    const float* qr = nullptr;
    const float *cr = nullptr, *sr = nullptr;
    if (active) {
      if (!p.decode) {
        qr = p.q + ((static_cast<size_t>(b) * p.S + qi) * p.H + head) * D;
        if (p.cos) {
          cr = p.cos + (static_cast<size_t>(b) * p.S + qi) * D;
          sr = p.sin + (static_cast<size_t>(b) * p.S + qi) * D;
        }
      } else {
        qr = p.q + (static_cast<size_t>(b) * p.H + head) * D;
        if (p.cos) {
          cr = p.cos + static_cast<size_t>(b) * D;
          sr = p.sin + static_cast<size_t>(b) * D;
        }
      }
    }
#pragma unroll
    for (int m = 0; m < DL; ++m) {
      const int d = e + 4 * m;
      float x = 0.f;
      if (active) {
        x = qr[d];
        if (cr) {
          const float rot = (d < D / 2) ? -qr[d + D / 2] : qr[d - D / 2];
          x = fmaf(x, cr[d], rot * sr[d]);
        }
      }
      qv[m] = x;
      acc[m] = 0.f;
    }
  }

  float m_run = -INFINITY, l_run = 0.f;
  const size_t kv_row_stride = p.decode ? D : static_cast<size_t>(p.Hkv) * D;
  const float* kbase = p.decode
                           ? p.k + (static_cast<size_t>(b) * p.Hkv + kvh) * p.L * D
                           : p.k + (static_cast<size_t>(b) * p.S * p.Hkv + kvh) * D;
  const float* vbase = p.decode
                           ? p.v + (static_cast<size_t>(b) * p.Hkv + kvh) * p.L * D
                           : p.v + (static_cast<size_t>(b) * p.S * p.Hkv + kvh) * D;
  const bool rotate_k = (!p.decode) && p.cos != nullptr;

  for (int j0 = 0; j0 < n_keys; j0 += KT) {
    __syncthreads();
    // ---- stage K (rotated) and V for keys [j0, j0 + KT).  128 is a multiple
    // of D, so a thread keeps one column d and takes every (128 / D)-th key;
    // the global loads of a batch of keys are all issued before any of them is
    // used, so a tile costs a few memory round trips rather than one per key.
    {
      constexpr int PER = KT * D / 128;  // tile elements per thread
      constexpr int BATCH = 8;
      constexpr int JSTEP = 128 / D;
      static_assert(128 % D == 0 && PER % BATCH == 0, "staging layout");
      const int d = tid % D, j_first = tid / D;
      const int dp = (d < D / 2) ? d + D / 2 : d - D / 2;  // rotation partner of d
      const bool lower = d < D / 2;
#pragma unroll 1
      for (int i0 = 0; i0 < PER; i0 += BATCH) {
        float kx[BATCH], kp[BATCH], cr[BATCH], sr[BATCH], vx[BATCH];
#pragma unroll
        for (int u = 0; u < BATCH; ++u) {
          const int key = j0 + j_first + (i0 + u) * JSTEP;
          kx[u] = kp[u] = cr[u] = sr[u] = vx[u] = 0.f;
          if (key < n_keys) {
            const float* kr = kbase + key * kv_row_stride;
            kx[u] = kr[d];
            vx[u] = vbase[key * kv_row_stride + d];
            if (rotate_k) {
              const size_t t = (static_cast<size_t>(b) * p.S + key) * D + d;
              kp[u] = kr[dp];
              cr[u] = p.cos[t];
              sr[u] = p.sin[t];
            }
          }
        }
#pragma unroll
        for (int u = 0; u < BATCH; ++u) {
          const int j = j_first + (i0 + u) * JSTEP;
          float k_out = kx[u];
          if (rotate_k) {
            const float rot = lower ? -kp[u] : kp[u];
            k_out = fmaf(kx[u], cr[u], rot * sr[u]);
          }
          ks[j][d] = k_out;
          vs[j][d] = vx[u];
        }
      }
    }
    __syncthreads();

    // ---- scores for this tile
    float s[KT];
    float tmax = -INFINITY;
#pragma unroll
    for (int j = 0; j < KT; ++j) {
      float dot = 0.f;
#pragma unroll
      for (int m = 0; m < DL; ++m) dot = fmaf(qv[m], ks[j][e + 4 * m], dot);
      dot += __shfl_xor_sync(0xffffffffu, dot, 1);
      dot += __shfl_xor_sync(0xffffffffu, dot, 2);
      const int key = j0 + j;
      float x = dot * p.scale;
      bool ok = active && key < n_keys && !(!p.decode && p.causal && key > qi);
      if (ok && p.mask) x += p.mask[(static_cast<size_t>(b) * p.S + qi) * p.S + key];
      x = ok ? x : -INFINITY;
      s[j] = x;
      tmax = fmaxf(tmax, x);
    }
    const float m_new = fmaxf(m_run, tmax);
    if (m_new == -INFINITY) continue;  // nothing visible yet for this row
    const float alpha = (m_run == -INFINITY) ? 0.f : expf(m_run - m_new);
    l_run *= alpha;
#pragma unroll
    for (int m = 0; m < DL; ++m) acc[m] *= alpha;
#pragma unroll
    for (int j = 0; j < KT; ++j) {
      const float pj = (s[j] == -INFINITY) ? 0.f : expf(s[j] - m_new);
      l_run += pj;
#pragma unroll
      for (int m = 0; m < DL; ++m) acc[m] = fmaf(pj, vs[j][e + 4 * m], acc[m]);
    }
    m_run = m_new;
  }

  if (!active) return;
  const float inv = (l_run > 0.f) ? 1.f / l_run : 0.f;
  float* orow = p.decode ? p.out + (static_cast<size_t>(b) * p.H + head) * D
                         : p.out + ((static_cast<size_t>(b) * p.S + qi) * p.H + head) * D;
#pragma unroll
  for (int m = 0; m < DL; ++m) orow[e + 4 * m] = acc[m] * inv;
}

}  // namespace la

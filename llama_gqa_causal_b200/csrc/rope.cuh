// RoPE kernels.
//
// * rope_table_kernel: cos/sin tables from position ids ("[HuggingFace
//   Transformers] LlamaAttention source walkthrough", section 2 step 3,
//   cos, sin = rotary_emb(x, position_ids); frequencies theta^(-2i/D) of the
//   RoFormer paper cited in "LLaMA2 large language model architecture
//   analysis", section "Rotary Position Encoding"; linear scaling divides the
//   position by the factor, "Llama2 Transformer architecture and optimisation
//   practice", section 6.1).  The angle is formed in fp64 and the table is
//   stored in fp32.
// * rope_rotate_bf16_kernel: x*cos + rotate_half(x)*sin applied once to every
//   K row of a prefill before the attention kernel streams K by TMA (fp32
//   arithmetic, one bf16 rounding of the result).
#pragma once
#include "common.cuh"

namespace la {

// Inverse frequencies theta^(-2i/D) formed on the host (in double) for
// head_dim <= 2 * kRopeHostFreqs, passed by value; 0 entries mean "form them
// on the device".
constexpr int kRopeHostFreqs = 64;
struct RopeFreqs {
  double inv[kRopeHostFreqs];
};

__global__ void rope_table_kernel(const long long* __restrict__ pos, long long n_rows, int D,
                                  double theta, double factor, float* __restrict__ cos_out,
                                  float* __restrict__ sin_out, const __grid_constant__ RopeFreqs freqs) {
  // blockDim.x is a multiple of D/2: each thread keeps one frequency index i
  // (so its inverse frequency is formed once) and walks the rows
  // a programmatic dependent launched after this kernel (a decode reading the
  // table) may be scheduled now; it waits for this grid to finish
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // this kernel is itself launched as a programmatic dependent of whatever
  // precedes it: the positions (and the table's own storage) are touched only
  // once that grid has finished
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int half = D / 2;
  const int i = static_cast<int>(threadIdx.x % half);
  const int rows_per_block = static_cast<int>(blockDim.x / half);
  const double inv_freq =
      half <= kRopeHostFreqs ? freqs.inv[i] : exp(-(2.0 * i / D) * log(theta));
  for (long long r = blockIdx.x * (long long)rows_per_block + threadIdx.x / half; r < n_rows;
       r += (long long)gridDim.x * rows_per_block) {
    const double angle = (static_cast<double>(pos[r]) / factor) * inv_freq;
    double s, c;
    sincos(angle, &s, &c);
    const float cf = static_cast<float>(c), sf = static_cast<float>(s);
    cos_out[r * D + i] = cf;
    cos_out[r * D + i + half] = cf;
    sin_out[r * D + i] = sf;
    sin_out[r * D + i + half] = sf;
  }
}

// x, y: [n_tokens, n_heads_x, D] bf16 (token = b * seq + s); cos/sin: [n_tokens, D].
// Each thread produces 8 output elements of the first half and the 8 matching
// elements of the second half of one row.
template <int D>
__global__ void rope_rotate_bf16_kernel(const __nv_bfloat16* __restrict__ x,
                                        __nv_bfloat16* __restrict__ y,
                                        const float* __restrict__ cos_t,
                                        const float* __restrict__ sin_t, long long n_tokens,
                                        int n_heads_x) {
  constexpr int HALF = D / 2;
  constexpr int CH = HALF / 8;  // 8-element chunks per half
  const long long total = n_tokens * n_heads_x * CH;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const int c = static_cast<int>(idx % CH);
    const long long row = idx / CH;              // token * n_heads_x + head
    const long long tok = row / n_heads_x;
    const __nv_bfloat16* xr = x + row * D;
    const uint4 a = *reinterpret_cast<const uint4*>(xr + c * 8);         // x[d], d < D/2
    const uint4 b = *reinterpret_cast<const uint4*>(xr + HALF + c * 8);  // x[d + D/2]
    const float* cr = cos_t + tok * D;
    const float* sr = sin_t + tok * D;
    const float4 c1a = *reinterpret_cast<const float4*>(cr + c * 8);
    const float4 c1b = *reinterpret_cast<const float4*>(cr + c * 8 + 4);
    const float4 c2a = *reinterpret_cast<const float4*>(cr + HALF + c * 8);
    const float4 c2b = *reinterpret_cast<const float4*>(cr + HALF + c * 8 + 4);
    const float4 s1a = *reinterpret_cast<const float4*>(sr + c * 8);
    const float4 s1b = *reinterpret_cast<const float4*>(sr + c * 8 + 4);
    const float4 s2a = *reinterpret_cast<const float4*>(sr + HALF + c * 8);
    const float4 s2b = *reinterpret_cast<const float4*>(sr + HALF + c * 8 + 4);
    const float c1[8] = {c1a.x, c1a.y, c1a.z, c1a.w, c1b.x, c1b.y, c1b.z, c1b.w};
    const float c2[8] = {c2a.x, c2a.y, c2a.z, c2a.w, c2b.x, c2b.y, c2b.z, c2b.w};
    const float s1[8] = {s1a.x, s1a.y, s1a.z, s1a.w, s1b.x, s1b.y, s1b.z, s1b.w};
    const float s2[8] = {s2a.x, s2a.y, s2a.z, s2a.w, s2b.x, s2b.y, s2b.z, s2b.w};
    const uint32_t au[4] = {a.x, a.y, a.z, a.w};
    const uint32_t bu[4] = {b.x, b.y, b.z, b.w};
    uint32_t lo[4], hi[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float x0 = bf16lo(au[e]), x1 = bf16hi(au[e]);  // first half, elements 2e, 2e+1
      const float z0 = bf16lo(bu[e]), z1 = bf16hi(bu[e]);  // second half
      // first half: x*cos - x[d+D/2]*sin ; second half: x[d+D/2]*cos + x*sin
      const float y0 = fmaf(x0, c1[2 * e], -z0 * s1[2 * e]);
      const float y1 = fmaf(x1, c1[2 * e + 1], -z1 * s1[2 * e + 1]);
      const float w0 = fmaf(z0, c2[2 * e], x0 * s2[2 * e]);
      const float w1 = fmaf(z1, c2[2 * e + 1], x1 * s2[2 * e + 1]);
      lo[e] = pack_bf16x2(y0, y1);
      hi[e] = pack_bf16x2(w0, w1);
    }
    __nv_bfloat16* yr = y + row * D;
    *reinterpret_cast<uint4*>(yr + c * 8) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    *reinterpret_cast<uint4*>(yr + HALF + c * 8) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
  }
}

}  // namespace la

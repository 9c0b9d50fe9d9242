// bf16 split-KV decode: one query token per sequence against a KV cache
// ("LLaMA2 large language model architecture analysis", section "KV cache":
// the new token's single query row attends to every cached key; section
// "GQA": several query heads share each K/V head, so one read of a K/V row
// serves the whole group).
//
// Work is the flattened list of 64-row chunks of every sequence, where a
// sequence is (batch entry, K/V head, chunk of <= 8 query heads of its group),
// built on the device from cache_lens.  A persistent grid (one CTA per SM)
// gives each CTA an even share of the chunks -- no two shares differ by more
// than one chunk -- and each CTA streams its K/V rows through a ring of TMA
// stages (64 rows of K and V each, 128-byte swizzle) without pausing at chunk
// or sequence boundaries.  The query slice and its cos/sin row are brought by
// bulk copy together with the first tile of each segment (a CTA's run of
// tiles inside one sequence).
//
// Four consumer warps take 16 rows of each stage:
//   S^T[16 keys x 8 heads]  = K[16 x D] . Q'^T[D x 8]    (mma m16n8k16; K by ldmatrix,
//                                                          Q' in registers)
//   O^T[D x 8 heads]       += V^T[D x 16] . P^T[16 x 8]   (V^T by ldmatrix.trans,
//                                                          P^T by movmatrix)
// so no tensor work is spent on padding when the group has 8 heads.  At the
// end of a segment the warps merge their running (max, sum, output) and write
// one partial: to the (batch, head) home slot when the segment starts at the
// sequence's first row, otherwise to the CTA's own slot (only a CTA's first
// segment can start inside a sequence).  decode_combine_kernel re-derives the
// segment boundaries from the chunk counts and merges with the log-sum-exp
// identity.
//
// Append mode (the decode step's own K/V row, "LLaMA2 large language model
// architecture analysis", section "KV cache": the new token's key and value
// join the cache before it is attended): the new token takes row
// p = min(len, L - 1) of its sequence; its key is rotated with the query's
// cos/sin row (the same position), both rows are written into the caches, and
// rows 0..p are attended.  The producer brings k_new, v_new (and cos/sin) with
// the tile that holds row p; the consumer warp that owns the row replaces the
// stale row in shared memory before using the tile, and the first head chunk
// of the sequence writes the row back to the caches.
#pragma once
#include "common.cuh"

namespace la {
namespace dec {
constexpr int TR = 64;           // cache rows per stage
constexpr int CH = 64;           // rows per work chunk (granule of the even split)
constexpr int NCW = 4;           // consumer warps (16 rows of a stage each)
constexpr int NSTAGE = 5;        // ring depth
constexpr int THREADS = (NCW + 1) * 32;
constexpr int MAX_BATCH = 4096;  // per-batch chunk prefix lives in shared memory
constexpr int MAX_CTAS = 256;    // persistent grid size cap (one CTA per SM)
// floats per partial row: D outputs, then max and sum; padded to 16 bytes
__host__ __device__ constexpr int part_stride(int d) { return d + 4; }
// Bytes of the workspace's last region: the chunk prefix over the batch
// ([bsz + 1] int32, written by the split kernel for the combine kernel).
__host__ __device__ inline size_t ws_prefix_bytes(int bsz) {
  return ((static_cast<size_t>(bsz) + 1) * 4 + 255) / 256 * 256;
}
}  // namespace dec

struct DecodeParams {
  const __nv_bfloat16* q;  // [b, H, D] un-rotated
  const float* cos;        // [b, D] or null
  const float* sin;
  const int* lens;         // [b]
  const __nv_bfloat16* k_new;  // append mode: [b, Hkv, D] un-rotated key of the new token
  const __nv_bfloat16* v_new;  // append mode: [b, Hkv, D]
  __nv_bfloat16* k_cache;      // append mode: the caches, written at row p
  __nv_bfloat16* v_cache;
  float* ws_home;          // [b, H, D + 4]: partial of the segment at a sequence's start
  float* ws_cta;           // [MAX_CTAS, 8, D + 4]: partial of a CTA's mid-sequence segment
  int* ws_prefix;          // [b + 1]: chunk prefix, written by CTA 0 for the combine kernel
  int bsz, H, Hkv, L, group, hchunks;
  float scale_log2;        // scale * log2(e)
};

// Per-stage description of the tile, written by the producer before it arms
// the stage's barrier.
struct DecTileMeta {
  int b, kvh, hc;
  int nvalid;      // rows of the tile below the sequence length (1..TR)
  int seg_start;   // first tile of a segment: consumers reset and read q
  int seg_end;     // last tile of a segment: consumers merge and write a partial
  int home;        // the segment starts at row 0 of its sequence
  int last;        // the CTA's final tile
  int new_row;     // append mode: row of the tile that holds the new token, else -1
  int new_pos;     // append mode: that row's index in the cache (p)
};

template <int D>
struct DecSmem {
  alignas(1024) __nv_bfloat16 k[dec::NSTAGE][dec::TR * D];
  alignas(1024) __nv_bfloat16 v[dec::NSTAGE][dec::TR * D];
  alignas(16) __nv_bfloat16 qv[dec::NSTAGE][8 * D];  // query slice at segment starts
  alignas(16) float cs[dec::NSTAGE][2 * D];            // cos row, sin row at segment starts
  alignas(16) __nv_bfloat16 kvn[dec::NSTAGE][2][D];    // append mode: k_new, v_new with their tile
  DecTileMeta meta[dec::NSTAGE];
  uint64_t full[dec::NSTAGE];
  uint64_t empty[dec::NSTAGE];
  float red_o[dec::NCW][8][D + 4];  // +4 spreads the merge's rows over the banks
  float red_m[dec::NCW][8];
  float red_l[dec::NCW][8];
  int chunk_prefix[dec::MAX_BATCH + 1];  // chunks per sequence of batch entries < b
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
// Untiled bulk copy global -> shared completing on an mbarrier
// (both addresses 16-byte aligned, size a multiple of 16).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ int clamp_len(int len, int L) { return len < 0 ? 0 : (len > L ? L : len); }
// Rows attended: the cached rows (clamped to [0, L]), or in append mode the
// cached rows before the new token's row p = min(len, L - 1) plus that row.
__device__ __forceinline__ int attend_len(int len, int L, int append) {
  return append ? clamp_len(len, L - 1) + 1 : clamp_len(len, L);
}

// Even split of n chunks over g CTAs: CTA i owns chunks [share_start(i), share_start(i + 1)).
__device__ __forceinline__ long long share_start(long long i, long long n, long long g) {
  return (i * n) / g;
}
// The CTA whose share holds chunk x: the largest i with share_start(i) <= x.
__device__ __forceinline__ long long share_owner(long long x, long long n, long long g) {
  return ((x + 1) * g + n - 1) / n - 1;
}

template <int D, bool APPEND>
__global__ void __launch_bounds__(dec::THREADS, 1) decode_bf16_kernel(
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
  const int per_b = p.Hkv * p.hchunks;  // sequences per batch entry
  if (warp == NCW && elect_one()) {  // descriptor fetch overlaps the prologue
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (threadIdx.x == 0) {  // shared memory only: set up before the grid-dependency wait
    for (int i = 0; i < NSTAGE; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], NCW);
    }
    fence_mbar_init();
  }
  // Launched as a programmatic dependent of whatever precedes it on the stream:
  // the CTAs may be resident before that grid has finished, so nothing in
  // global memory is read or written before this wait (the previous decode's
  // combine still reads the workspace this kernel writes).
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // ---- chunk counts per batch entry, prefix-summed (identical in every CTA):
  // each thread sums a contiguous run of entries, the run totals are scanned
  // with warp shuffles and the per-warp totals, then each thread writes the
  // prefixes of its run
  {
    __shared__ int warp_total[THREADS / 32];
    const int per = (p.bsz + THREADS - 1) / THREADS;
    const int lo = min(p.bsz, static_cast<int>(threadIdx.x) * per), hi = min(p.bsz, lo + per);
    int sum = 0;
    for (int b = lo; b < hi; ++b) sum += (attend_len(p.lens[b], p.L, APPEND) + CH - 1) / CH;
    int incl = sum;  // inclusive scan of the run totals within the warp
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) warp_total[warp] = incl;
    __syncthreads();
    int acc = incl - sum;  // exclusive prefix of this thread's run
    for (int w = 0; w < warp; ++w) acc += warp_total[w];
    if (threadIdx.x == THREADS - 1) s.chunk_prefix[p.bsz] = acc + sum;
    for (int b = lo; b < hi; ++b) {
      s.chunk_prefix[b] = acc;
      acc += (attend_len(p.lens[b], p.L, APPEND) + CH - 1) / CH;
    }
    __syncthreads();
    // the combine kernel reads the prefix once this grid has finished
    if (blockIdx.x == 0)
      for (int b = threadIdx.x; b <= p.bsz; b += THREADS) p.ws_prefix[b] = s.chunk_prefix[b];
  }
  // the combine kernel may be scheduled now; it waits for this grid to finish
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const long long n_chunks = static_cast<long long>(s.chunk_prefix[p.bsz]) * per_b;
  const long long x0 = share_start(blockIdx.x, n_chunks, gridDim.x);
  const long long x1 = share_start(blockIdx.x + 1, n_chunks, gridDim.x);
  if (x0 >= x1) return;  // uniform across the CTA: no share

  if (warp == NCW) {  // ---------------------------------------------- TMA producer
    // batch entry of the share's first chunk: the largest b with
    // chunk_prefix[b] * per_b <= x0, by binary search (a scan from entry 0
    // would delay the first copies of the last CTAs by up to bsz steps of
    // dependent shared-memory loads)
    int b = 0;
    {
      int hi = p.bsz - 1;
      while (b < hi) {
        const int mid = (b + hi + 1) >> 1;
        if (static_cast<long long>(s.chunk_prefix[mid]) * per_b <= x0) b = mid;
        else hi = mid - 1;
      }
    }
    int it = 0;  // tiles issued
    bool ok = true;
    bool home = false;
    for (long long x = x0; x < x1 && ok; ++x) {
      // global chunk x -> batch entry b, sequence (kvh, hc) within b, chunk c
      while (static_cast<long long>(s.chunk_prefix[b + 1]) * per_b <= x) ++b;
      const int nch_b = s.chunk_prefix[b + 1] - s.chunk_prefix[b];
      const long long xb = x - static_cast<long long>(s.chunk_prefix[b]) * per_b;
      const int seq = static_cast<int>(xb / nch_b);
      const int c = static_cast<int>(xb - static_cast<long long>(seq) * nch_b);
      const int kvh = seq / p.hchunks, hc = seq - kvh * p.hchunks;
      const int len = attend_len(p.lens[b], p.L, APPEND);
      const bool first_chunk_of_seg = (x == x0) || (c == 0);
      const bool last_chunk_of_seg = (x + 1 == x1) || (c + 1 == nch_b);
      if (first_chunk_of_seg) home = (c == 0);
      const int row_end = min(len, (c + 1) * CH);
      for (int row0 = c * CH; row0 < row_end; row0 += TR, ++it) {
        const int st = it % NSTAGE;
        if (it >= NSTAGE && !mbar_wait(&s.empty[st], ((it / NSTAGE) - 1) & 1)) {
          ok = false;
          break;
        }
        const bool seg_start = first_chunk_of_seg && row0 == c * CH;
        const bool tile_last_of_chunk = row0 + TR >= row_end;
        if (elect_one()) {
          DecTileMeta& m = s.meta[st];
          m.b = b;
          m.kvh = kvh;
          m.hc = hc;
          m.nvalid = min(TR, row_end - row0);
          m.seg_start = seg_start;
          m.seg_end = last_chunk_of_seg && tile_last_of_chunk;
          m.home = home;
          m.last = (x + 1 == x1) && tile_last_of_chunk;
          // append mode: the new token is the sequence's last row
          const bool has_new = APPEND && row0 <= len - 1 && len - 1 < row0 + TR;
          m.new_row = has_new ? len - 1 - row0 : -1;
          m.new_pos = len - 1;
          const bool need_cs = p.cos != nullptr && (seg_start || has_new);
          const int nh = min(8, p.group - hc * 8);
          uint32_t bytes = 2u * TR * D * 2u;
          if (seg_start) bytes += nh * D * 2u;
          if (need_cs) bytes += 2u * D * 4u;
          if (has_new) bytes += 2u * D * 2u;
          mbar_arrive_expect_tx(&s.full[st], bytes);
          const int bh = b * p.Hkv + kvh;
#pragma unroll
          for (int cb = 0; cb < CB; ++cb) {
            tma_load_3d(&s.k[st][cb * TR * 64], &tm_k, &s.full[st], cb * 64, row0, bh);
            tma_load_3d(&s.v[st][cb * TR * 64], &tm_v, &s.full[st], cb * 64, row0, bh);
          }
          if (seg_start)
            bulk_load(&s.qv[st][0], p.q + (static_cast<size_t>(b) * p.H + kvh * p.group + hc * 8) * D,
                      nh * D * 2u, &s.full[st]);
          if (need_cs) {
            bulk_load(&s.cs[st][0], p.cos + static_cast<size_t>(b) * D, D * 4u, &s.full[st]);
            bulk_load(&s.cs[st][D], p.sin + static_cast<size_t>(b) * D, D * 4u, &s.full[st]);
          }
          if (has_new) {
            bulk_load(&s.kvn[st][0][0], p.k_new + static_cast<size_t>(bh) * D, D * 2u, &s.full[st]);
            bulk_load(&s.kvn[st][1][0], p.v_new + static_cast<size_t>(bh) * D, D * 2u, &s.full[st]);
          }
        }
        __syncwarp();
      }
    }
    // never leave with copies in flight: wait for the last issued stages to land
    for (int i = max(0, it - NSTAGE); i < it; ++i)
      if (!mbar_wait(&s.full[i % NSTAGE], (i / NSTAGE) & 1)) break;
    return;
  }

  // ------------------------------------------------------------------ consumers
  const int g = lane >> 2, t = lane & 3;
  const int mat = lane >> 3, r8 = lane & 7;
  uint32_t qf[KSTEPS][2];
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
  float o[KSTEPS][4];
#pragma unroll
  for (int mt = 0; mt < KSTEPS; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
#pragma unroll
  for (int kk = 0; kk < KSTEPS; ++kk) qf[kk][0] = qf[kk][1] = 0u;
  for (int it = 0;; ++it) {
    const int st = it % NSTAGE;
    if (!mbar_wait(&s.full[st], (it / NSTAGE) & 1)) break;
    const DecTileMeta m = s.meta[st];
    if (m.seg_start) {
      m_run[0] = m_run[1] = -INFINITY;
      l_run[0] = l_run[1] = 0.f;
#pragma unroll
      for (int mt = 0; mt < KSTEPS; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
      // Q' fragments: lane holds head g of the chunk, dims kk*16 + 2t + {0, 1, 8, 9}.
      // The rotation partner of dim d is d +- D/2, i.e. k-step kk +- D/32, same lane.
      const bool hvalid = m.hc * 8 + g < p.group;
      float qx[KSTEPS][4];
#pragma unroll
      for (int kk = 0; kk < KSTEPS; ++kk)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const int d = kk * 16 + 2 * t + (jj < 2 ? jj : jj + 6);
          qx[kk][jj] = hvalid ? __bfloat162float(s.qv[st][g * D + d]) : 0.f;
        }
#pragma unroll
      for (int kk = 0; kk < KSTEPS; ++kk) {
        float y[4];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          y[jj] = qx[kk][jj];
          if (p.cos != nullptr) {
            const int d = kk * 16 + 2 * t + (jj < 2 ? jj : jj + 6);
            const float rot = (kk < KSTEPS / 2) ? -qx[kk + KSTEPS / 2][jj] : qx[kk - KSTEPS / 2][jj];
            y[jj] = fmaf(qx[kk][jj], s.cs[st][d], rot * s.cs[st][D + d]);
          }
        }
        qf[kk][0] = pack_bf16x2(y[0], y[1]);
        qf[kk][1] = pack_bf16x2(y[2], y[3]);
      }
    }
    if (APPEND && m.new_row >= 0 && (m.new_row >> 4) == warp) {
      // append mode: this warp's rows hold the new token.  Replace the stale
      // row of the stage by the rotated k_new and by v_new (same 128-byte
      // swizzle as the TMA tile), and let the first head chunk of the sequence
      // write both rows into the caches.
      const int r = m.new_row;
      uint8_t* kb = reinterpret_cast<uint8_t*>(&s.k[st][0]);
      uint8_t* vb = reinterpret_cast<uint8_t*>(&s.v[st][0]);
      const size_t crow = (static_cast<size_t>(m.b * p.Hkv + m.kvh) * p.L + m.new_pos) * D;
      auto at = [&](int dd) {
        return (dd / 64) * STAGE_BLOCK_BYTES + sw128_offset(r, (dd % 64) / 8) + (dd % 8) * 2;
      };
      for (int i = lane; i < D / 2; i += 32) {
        const int d1 = i, d2 = i + D / 2;
        const float x = __bfloat162float(s.kvn[st][0][d1]), z = __bfloat162float(s.kvn[st][0][d2]);
        float k1 = x, k2 = z;
        if (p.cos != nullptr) {
          k1 = fmaf(x, s.cs[st][d1], -z * s.cs[st][D + d1]);
          k2 = fmaf(z, s.cs[st][d2], x * s.cs[st][D + d2]);
        }
        const __nv_bfloat16 kr1 = __float2bfloat16_rn(k1), kr2 = __float2bfloat16_rn(k2);
        const __nv_bfloat16 v1 = s.kvn[st][1][d1], v2 = s.kvn[st][1][d2];
        *reinterpret_cast<__nv_bfloat16*>(kb + at(d1)) = kr1;
        *reinterpret_cast<__nv_bfloat16*>(kb + at(d2)) = kr2;
        *reinterpret_cast<__nv_bfloat16*>(vb + at(d1)) = v1;
        *reinterpret_cast<__nv_bfloat16*>(vb + at(d2)) = v2;
        if (m.hc == 0) {
          p.k_cache[crow + d1] = kr1;
          p.k_cache[crow + d2] = kr2;
          p.v_cache[crow + d1] = v1;
          p.v_cache[crow + d2] = v2;
        }
      }
      __syncwarp();
    }
    const int nvalid = min(16, m.nvalid - warp * 16);
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
          *reinterpret_cast<uint4*>(vb + (rem / 8) * STAGE_BLOCK_BYTES + sw128_offset(rr, rem % 8)) =
              make_uint4(0, 0, 0, 0);
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
        ldsm_x4(kbase + (col / 64) * STAGE_BLOCK_BYTES + sw128_offset(krow, (col % 64) / 8), a0, a1,
                a2, a3);
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
        const float m_new = fmaxf(m_run[h], mx);  // finite: this warp has a valid key
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
        ldsm_x4_t(vbase + (col / 64) * STAGE_BLOCK_BYTES + sw128_offset(vrow, (col % 64) / 8), a0,
                  a1, a2, a3);
        mma_bf16_16816(o[mt], a0, a1, a2, a3, pb0, pb1);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.empty[st]);

    if (m.seg_end) {
      // ---- merge the four warps' partial states, write the segment's partial
      float lr[2] = {l_run[0], l_run[1]};
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        lr[h] += __shfl_xor_sync(0xffffffffu, lr[h], 4);
        lr[h] += __shfl_xor_sync(0xffffffffu, lr[h], 8);
        lr[h] += __shfl_xor_sync(0xffffffffu, lr[h], 16);
      }
      if (g == 0) {
        s.red_m[warp][2 * t] = m_run[0];
        s.red_m[warp][2 * t + 1] = m_run[1];
        s.red_l[warp][2 * t] = lr[0];
        s.red_l[warp][2 * t + 1] = lr[1];
      }
#pragma unroll
      for (int mt = 0; mt < KSTEPS; ++mt) {
        s.red_o[warp][2 * t][mt * 16 + g] = o[mt][0];
        s.red_o[warp][2 * t + 1][mt * 16 + g] = o[mt][1];
        s.red_o[warp][2 * t][mt * 16 + g + 8] = o[mt][2];
        s.red_o[warp][2 * t + 1][mt * 16 + g + 8] = o[mt][3];
      }
      named_bar_sync(1, NCW * 32);
      {
        constexpr int PER = D / 16;  // dims per thread: 128 threads cover 8 heads x D
        const int tid = threadIdx.x;
        const int hh = tid >> 4;
        const int d0 = (tid & 15) * PER;
        if (m.hc * 8 + hh < p.group) {
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
          const int head = m.kvh * p.group + m.hc * 8 + hh;
          float* dst = m.home
              ? p.ws_home + (static_cast<size_t>(m.b) * p.H + head) * part_stride(D)
              : p.ws_cta + (static_cast<size_t>(blockIdx.x) * 8 + hh) * part_stride(D);
#pragma unroll
          for (int i = 0; i < PER; i += 4) {
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int w = 0; w < NCW; ++w) {
              acc.x = fmaf(f[w], s.red_o[w][hh][d0 + i], acc.x);
              acc.y = fmaf(f[w], s.red_o[w][hh][d0 + i + 1], acc.y);
              acc.z = fmaf(f[w], s.red_o[w][hh][d0 + i + 2], acc.z);
              acc.w = fmaf(f[w], s.red_o[w][hh][d0 + i + 3], acc.w);
            }
            *reinterpret_cast<float4*>(dst + d0 + i) = acc;
          }
          if ((tid & 15) == 0) {
            dst[D] = mstar;
            dst[D + 1] = lsum;
          }
        }
      }
      named_bar_sync(1, NCW * 32);  // red_* are reused by the next segment
    }
    if (m.last) break;
  }
}

// Merge the partials of the heads of one sequence (batch entry, K/V head,
// chunk of <= 8 query heads): one warp per head, each lane D/32 dimensions.
// The sequence's segments start at its first chunk (home slot) and at every
// chunk where some CTA's share begins inside it (that CTA's own slot).
//   m* = max_s m_s,  l = sum_s l_s 2^(m_s - m*),  o = sum_s o_s 2^(m_s - m*) / l.
// The chunk prefix of the batch comes from the split kernel through the
// workspace and, like everything else that grid wrote, is read only after the
// wait for it; the partials of up to kEager segments are then loaded at once.
namespace dec {
constexpr int COMBINE_THREADS = 256;  // 8 warps = the heads of one sequence
}
template <int D>
__global__ void __launch_bounds__(dec::COMBINE_THREADS) decode_combine_kernel(
    const float* ws_home, const float* ws_cta, const int* ws_prefix,
    __nv_bfloat16* __restrict__ out, int bsz, int H, int Hkv, int group, int hchunks,
    int n_ctas) {
  constexpr int kEager = 4;
  constexpr int VEC = D / 32;  // dimensions per lane
  const int seq = blockIdx.x, b = blockIdx.y;
  const int kvh = seq / hchunks, hc = seq - kvh * hchunks;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // a programmatic dependent launched after this kernel (the next decode) may
  // be scheduled now; it waits for this grid to finish before touching memory
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // the split kernel's writes (prefix and partials) are visible after this
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const long long prefix_b = ws_prefix[b];
  const long long total = ws_prefix[bsz];
  const int per_b = Hkv * hchunks;
  const int nch = static_cast<int>(ws_prefix[b + 1] - prefix_b);
  const long long n_chunks = total * per_b;
  const long long G = n_ctas;
  const long long P = prefix_b * per_b + static_cast<long long>(seq) * nch;
  // owners of the CTA shares that begin strictly inside [P, P + nch); equal
  // starts mean empty shares, and the owner of a start is the last CTA with it
  long long gi = (nch > 0) ? share_owner(P, n_chunks, G) + 1 : G;
  long long last_start = P;
  auto next_owner = [&]() -> long long {
    for (; gi < G; ++gi) {
      const long long st = share_start(gi, n_chunks, G);
      if (st >= P + nch) break;
      if (st == last_start) continue;
      last_start = st;
      ++gi;
      return share_owner(st, n_chunks, G);
    }
    gi = G;
    return -1;
  };
  long long own[kEager];
#pragma unroll
  for (int k = 0; k < kEager; ++k) own[k] = next_owner();

  const int hq = hc * 8 + warp;  // query head within the group
  if (hq >= group) return;
  const int head = kvh * group + hq;
  float mstar = -INFINITY, lsum = 0.f, acc[VEC];
#pragma unroll
  for (int v = 0; v < VEC; ++v) acc[v] = 0.f;
  auto add = [&](float mc, float lc, const float (&oc)[VEC]) {
    const float m_new = fmaxf(mstar, mc);
    const float fo = (mstar == -INFINITY) ? 0.f : ex2_approx(mstar - m_new);
    const float fc = ex2_approx(mc - m_new);
    lsum = lsum * fo + lc * fc;
#pragma unroll
    for (int v = 0; v < VEC; ++v) acc[v] = acc[v] * fo + oc[v] * fc;
    mstar = m_new;
  };
  auto load = [&](const float* part, float& m, float& l, float (&o)[VEC]) {
    m = part[D];
    l = part[D + 1];
#pragma unroll
    for (int v = 0; v < VEC; v += 2) {
      const float2 x = *reinterpret_cast<const float2*>(part + lane * VEC + v);
      o[v] = x.x;
      o[v + 1] = x.y;
    }
  };
  if (nch > 0) {
    float pm[kEager + 1], pl[kEager + 1], po[kEager + 1][VEC];
    load(ws_home + (static_cast<size_t>(b) * H + head) * dec::part_stride(D), pm[0], pl[0], po[0]);
#pragma unroll
    for (int k = 0; k < kEager; ++k)
      if (own[k] >= 0)
        load(ws_cta + (static_cast<size_t>(own[k]) * 8 + warp) * dec::part_stride(D), pm[k + 1],
             pl[k + 1], po[k + 1]);
    add(pm[0], pl[0], po[0]);
#pragma unroll
    for (int k = 0; k < kEager; ++k)
      if (own[k] >= 0) add(pm[k + 1], pl[k + 1], po[k + 1]);
    // sequences split over more CTAs than that (short batches): the rest one by one
    if (own[kEager - 1] >= 0) {
      for (long long ow = next_owner(); ow >= 0; ow = next_owner()) {
        float m, l, o[VEC];
        load(ws_cta + (static_cast<size_t>(ow) * 8 + warp) * dec::part_stride(D), m, l, o);
        add(m, l, o);
      }
    }
  }
  const float inv = (lsum > 0.f) ? 1.f / lsum : 0.f;
  __nv_bfloat16* dst = out + (static_cast<size_t>(b) * H + head) * D + lane * VEC;
#pragma unroll
  for (int v = 0; v < VEC; v += 2)
    *reinterpret_cast<uint32_t*>(dst + v) = pack_bf16x2(acc[v] * inv, acc[v + 1] * inv);
}

}  // namespace la

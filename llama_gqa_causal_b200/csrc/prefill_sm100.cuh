// bf16 prefill attention on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// Computes, for each query head h and query position i,
//   out[b, i, h*D:(h+1)*D] = softmax_j(scale * q'_i . k'_j + mask_ij) v_j
// ("[HuggingFace Transformers] LlamaAttention source walkthrough", section
// 1.2 steps 2-4 and section 2 steps 3-6), with j <= i when causal, K/V head
// h / group (repeat_kv, step 4), fp32 scores and softmax (step 5.2) and the
// probabilities rounded to bf16 before the product with V (the `.to(dtype)`
// of step 5.2).
//
// Work unit: a Q tile = 128 consecutive query positions of one query head.
// The Q tiles of one (batch, K/V head) are ordered position-block-major, so
// consecutive units are the heads of one GQA group at the same positions (or,
// with group 1, consecutive position blocks).  A CTA owns two consecutive
// units and streams each K/V tile of 128 keys through shared memory once for
// both; causal tiles past a unit's last position are skipped.
//
// Warp roles (384 threads = three warpgroups):
//   warp 0      TMA producer: K' and V tiles (2 stages each), 128B swizzle
//   warp 1      TMEM allocator and MMA issuer (one thread):
//                 S_t = Q_t K_j^T   (SS: both operands K-major in smem)
//                 O_t += P_t V_j    (TS: P from TMEM, V MN-major in smem)
//   warps 2-3   idle (complete warpgroup 0, which gives registers away)
//   warps 4-7   softmax of unit 0, warps 8-11 softmax of unit 1: each thread
//               owns one query row (= one TMEM lane; warp w reaches the 32
//               lanes of quarter w % 4).  Before the loop they
//               rotate their Q row with RoPE and write it to shared memory
//               (this is the "RoPE while staging Q" step); K arrives already
//               rotated (a separate pass rotates each K row exactly once).
// TMEM (512 columns): S_0, S_1 (128 fp32 columns each), O_0, O_1 (D each).
// P_t (bf16, two per column) is written over the first 64 columns of S_t:
// the MMA warp issues the next S_t = Q_t K^T only after O_t += P_t V in the
// same tcgen05 issue order, so the overwrite follows the read.
// Rescaling of O is lazy: the running max used for the exponentials moves
// only when a row's max grows by more than 2^8, which keeps O corrections rare.
// Epilogue: O / l in bf16 is staged in the Q tile buffer and stored by TMA.
//
// Instances (template flags, so each compiles only its own bookkeeping):
//   WINDOW          causal sliding window: a unit starts at the K/V tile of its
//                   first row's window start; window-edge tiles are masked
//   VARLEN == 1     right-padded batch: per-entry lengths; padded keys masked,
//                   padded V rows zeroed in the stage, padded rows output zero
//   VARLEN == 2     packed sequences: as 1, with each sequence addressed from
//                   its first token and its rows stored by their own threads
#pragma once
#include <type_traits>

#include "common.cuh"

namespace la {
namespace pf {
constexpr int BM = 128;       // query rows per tile (= TMEM lanes)
constexpr int BN = 128;       // keys per K/V tile
constexpr int NQ = 2;         // Q tiles (units) per CTA
#ifndef LA_PF_KSTAGES
#define LA_PF_KSTAGES 2
#endif
#ifndef LA_PF_VSTAGES
#define LA_PF_VSTAGES 2
#endif
constexpr int KSTAGES = LA_PF_KSTAGES;  // K tile ring depth
constexpr int VSTAGES = LA_PF_VSTAGES;  // V tile ring depth
constexpr int THREADS = 384;  // warpgroup 0: TMA + MMA warps; warpgroups 1, 2: softmax
// Register budget per warpgroup after setmaxnreg.  setmaxnreg.inc can only
// take registers that the block was launched with: 384 threads x 168 (the
// most __launch_bounds__(384, 1) allows), i.e. 504 per lane over the three
// warpgroups that share an SMSP: 56 + 224 + 224.  A split above that makes the
// increasing warps wait for registers that never come free, so it is refused
// here.
constexpr int kRegsControl = 56;
constexpr int kRegsSoftmax = 224;
constexpr int kRegsAtLaunch = (65536 / THREADS) / 8 * 8;  // 168
static_assert(kRegsControl % 8 == 0 && kRegsSoftmax % 8 == 0, "setmaxnreg takes multiples of 8");
static_assert(kRegsControl + 2 * kRegsSoftmax <= 3 * kRegsAtLaunch,
              "setmaxnreg split exceeds the registers the block is launched with");
constexpr float kRescaleThreshold = 8.0f;  // log2 units
// Of every 8 consecutive pairs of probabilities in an interior tile, this
// many are exponentiated on the FMA pipe (exp2_poly2), the rest on MUFU.
#ifndef LA_POLY_PAIRS_OF_8
#define LA_POLY_PAIRS_OF_8 3
#endif
constexpr int kPolyPairsOf8 = LA_POLY_PAIRS_OF_8;
// Pairs of the second P half exponentiated before the wait for the first
// half's TMEM store.
#ifndef LA_PF_ST_OVERLAP
#define LA_PF_ST_OVERLAP 8
#endif
constexpr int kStOverlap = LA_PF_ST_OVERLAP;
}  // namespace pf

struct PrefillParams {
  const __nv_bfloat16* q;  // [b, S, H, D]
  const float* cos;        // [b, S, D] or null
  const float* sin;
  const float* mask;       // [b, 1, S, S] or null
  __nv_bfloat16* out;      // [b, S, H*D]
  int bsz, H, Hkv, S, group;
  int n_pb;                // ceil(S / BM)
  int n_kb;                // ceil(S / BN)
  int ctas_per_kvh;        // ceil(group * n_pb / 2)
  int bkv_per_bundle;      // (batch, K/V head) pairs scheduled together (their K/V fit in L2)
  int causal;
  int window;              // sliding-window instance: query i sees keys i - window < j <= i
  const int* seq_lens;     // padded variable-length instance: [b] valid rows of each batch entry
  const int* cu_seqlens;   // packed instance: [b + 1] first token of each sequence
  int T;                   // packed instance: tokens in the packed tensors
  float scale_log2;        // scale * log2(e)
};

template <int D>
struct PfSmem {
  alignas(1024) __nv_bfloat16 q[pf::NQ][pf::BM * D];
  alignas(1024) __nv_bfloat16 k[pf::KSTAGES][pf::BN * D];
  alignas(1024) __nv_bfloat16 v[pf::VSTAGES][pf::BN * D];
  uint64_t k_full[pf::KSTAGES], k_empty[pf::KSTAGES];
  uint64_t v_full[pf::VSTAGES], v_empty[pf::VSTAGES];
  uint64_t q_loaded[pf::NQ], q_ready[pf::NQ], s_full[pf::NQ], p_lo[pf::NQ], p_hi[pf::NQ];
  uint64_t o_full[pf::NQ];
  uint64_t mma_done;
  uint32_t tmem_base;
};

template <int D, bool WINDOW, int VARLEN>
__global__ void __launch_bounds__(pf::THREADS, 1)
    prefill_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v,
                         const __grid_constant__ CUtensorMap tm_out, PrefillParams p) {
  using namespace pf;
  constexpr int CB = D / 64;                       // 64-column swizzle blocks per row
  constexpr uint32_t BLOCK_BYTES = BM * 128;       // one [128 rows x 64 cols] bf16 block
  constexpr uint32_t TILE_BYTES = BM * D * 2;
  constexpr uint32_t IDESC_QK = idesc_bf16(BM, BN, false);
  constexpr uint32_t IDESC_PV = idesc_bf16(BM, D, true);
  constexpr uint32_t TMEM_COLS = 512;

  extern __shared__ uint8_t smem_raw[];
  PfSmem<D>& s = *reinterpret_cast<PfSmem<D>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- work decomposition.  The (batch, K/V head) pairs are taken in bundles
  // whose K/V fit in L2 together, so the CTAs that share a K/V head run close
  // in time and its tiles are read from DRAM about once; inside a bundle, heavy
  // (late position block) CTAs go first, over all of the bundle's pairs.
  const int n_bkv = p.bsz * p.Hkv;
  const int nb = p.bkv_per_bundle;
  const int bundle = blockIdx.x / (nb * p.ctas_per_kvh);
  const int bsize = min(nb, n_bkv - bundle * nb);  // the last bundle may be smaller
  const int local = blockIdx.x - bundle * nb * p.ctas_per_kvh;
  const int rank = local / bsize;
  const int bkv = bundle * nb + (local - rank * bsize);
  const int b = bkv / p.Hkv, kvh = bkv - (bkv / p.Hkv) * p.Hkv;
  const int cta = p.ctas_per_kvh - 1 - rank;
  // two units per CTA, kept in scalars (never in arrays indexed at run time)
  const int n_units = p.group * p.n_pb;
  const int u0 = cta * NQ, u1 = cta * NQ + 1;
  const int pb0 = u0 / p.group, pb1 = u1 / p.group;
  const int head0 = kvh * p.group + (u0 - pb0 * p.group);
  const int head1 = kvh * p.group + (u1 - pb1 * p.group);
  // variable length (VARLEN 1: right-padded batch; 2: packed sequences): entry
  // b holds S_b valid rows (queries and keys).  Padded rows are never attended
  // and their outputs are zero; in the packed layout the rows past S_b are the
  // next sequence's, never attended and never written.  Packed sequence b
  // starts at token tok0 of tensors with a batch extent of one.
  const int tok0 = (VARLEN == 2) ? min(max(p.cu_seqlens[b], 0), p.T) : 0;
  const int S_b = (VARLEN == 1)   ? min(max(p.seq_lens[b], 0), p.S)
                  : (VARLEN == 2) ? min(max(p.cu_seqlens[b + 1] - tok0, 0), min(p.S, p.T - tok0))
                                  : p.S;
  const int bco = (VARLEN == 2) ? 0 : b;  // batch coordinate of the tensor maps
  const int n_kb_b = VARLEN ? (S_b + BN - 1) / BN : p.n_kb;
  auto n_tiles = [&](int pb) {
    if (VARLEN && pb * BM >= S_b) return 0;  // every row of the Q tile is padding
    return p.causal ? min(n_kb_b, ((pb + 1) * BM + BN - 1) / BN) : n_kb_b;
  };
  const int nkv0 = (u0 < n_units) ? n_tiles(pb0) : 0;
  const int nkv1 = (u1 < n_units) ? n_tiles(pb1) : 0;
  const int n_max = max(nkv0, nkv1);
  // sliding window: a unit's first K/V tile is the one holding key
  // pb * BM - window + 1 (the window start of its first row); the CTA streams
  // tiles j_min .. n_max - 1, the union of its units' ranges (contiguous: the
  // two units' position blocks differ by at most one)
  auto first_tile = [&](int pb) { return WINDOW ? max(0, pb * BM - p.window + 1) / BN : 0; };
  const int jlo0 = first_tile(pb0);
  const int jlo1 = nkv1 > 0 ? first_tile(pb1) : jlo0;
  const int j_min = min(jlo0, jlo1);
  const int n_it = n_max - j_min;  // tiles streamed

  // ---- setup
  if (threadIdx.x == 0) {
    for (int i = 0; i < KSTAGES; ++i) { mbar_init(&s.k_full[i], 1); mbar_init(&s.k_empty[i], 1); }
    for (int i = 0; i < VSTAGES; ++i) { mbar_init(&s.v_full[i], 1); mbar_init(&s.v_empty[i], 1); }
    for (int t = 0; t < NQ; ++t) {
      mbar_init(&s.q_loaded[t], 1);
      mbar_init(&s.q_ready[t], 4);
      mbar_init(&s.s_full[t], 1);
      mbar_init(&s.p_lo[t], 4);
      mbar_init(&s.p_hi[t], 4);
      mbar_init(&s.o_full[t], 1);
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
  // TMEM columns: S_0 [0,128), S_1 [128,256), O_0 [256,256+D), O_1 [256+D,256+2D)
  auto tm_s = [&](int t) { return tmem + static_cast<uint32_t>(t * BN); };
  auto tm_o = [&](int t) { return tmem + static_cast<uint32_t>(2 * BN + t * D); };
  if (warp == 0) {
    // ================================================================ TMA producer
    // The whole warp runs the loop (waits and addresses stay warp-uniform);
    // one elected lane issues the copies.
    setmaxnreg_dec<kRegsControl>();
    if (elect_one()) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_out);
      // the two Q tiles (raw; rotated in shared memory by their softmax warps)
      if (nkv0 > 0) {
        mbar_arrive_expect_tx(&s.q_loaded[0], TILE_BYTES);
#pragma unroll
        for (int cb = 0; cb < CB; ++cb)
          tma_load_4d(reinterpret_cast<uint8_t*>(&s.q[0][0]) + cb * BLOCK_BYTES, &tm_q,
                      &s.q_loaded[0], cb * 64, head0, tok0 + pb0 * BM, bco);
      }
      if (nkv1 > 0) {
        mbar_arrive_expect_tx(&s.q_loaded[1], TILE_BYTES);
#pragma unroll
        for (int cb = 0; cb < CB; ++cb)
          tma_load_4d(reinterpret_cast<uint8_t*>(&s.q[1][0]) + cb * BLOCK_BYTES, &tm_q,
                      &s.q_loaded[1], cb * 64, head1, tok0 + pb1 * BM, bco);
      }
    }
    __syncwarp();
    int k_issued = 0, v_issued = 0;
    for (int it = 0; it < n_it; ++it) {
      const int j = j_min + it;  // K/V tile
      const int ks = it % KSTAGES;
      if (it >= KSTAGES && !mbar_wait(&s.k_empty[ks], ((it / KSTAGES) - 1) & 1)) break;
      if (elect_one()) {
        mbar_arrive_expect_tx(&s.k_full[ks], TILE_BYTES);
#pragma unroll
        for (int cb = 0; cb < CB; ++cb)
          tma_load_4d(reinterpret_cast<uint8_t*>(&s.k[ks][0]) + cb * BLOCK_BYTES, &tm_k,
                      &s.k_full[ks], cb * 64, kvh, tok0 + j * BN, bco);
      }
      __syncwarp();
      k_issued = it + 1;
      const int vs = it % VSTAGES;
      if (it >= VSTAGES && !mbar_wait(&s.v_empty[vs], ((it / VSTAGES) - 1) & 1)) break;
      if (elect_one()) {
        mbar_arrive_expect_tx(&s.v_full[vs], TILE_BYTES);
#pragma unroll
        for (int cb = 0; cb < CB; ++cb)
          tma_load_4d(reinterpret_cast<uint8_t*>(&s.v[vs][0]) + cb * BLOCK_BYTES, &tm_v,
                      &s.v_full[vs], cb * 64, kvh, tok0 + j * BN, bco);
      }
      __syncwarp();
      v_issued = it + 1;
    }
    // leave no copy in flight
    if (nkv0 > 0) mbar_wait(&s.q_loaded[0], 0);
    if (nkv1 > 0) mbar_wait(&s.q_loaded[1], 0);
    for (int j = max(0, k_issued - KSTAGES); j < k_issued; ++j)
      if (!mbar_wait(&s.k_full[j % KSTAGES], (j / KSTAGES) & 1)) break;
    for (int j = max(0, v_issued - VSTAGES); j < v_issued; ++j)
      if (!mbar_wait(&s.v_full[j % VSTAGES], (j / VSTAGES) & 1)) break;
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    // Converged warp, single elected issuing lane (tcgen05.mma and commit
    // take warp-uniform operands).
    setmaxnreg_dec<kRegsControl>();
    bool ok = true;
    const uint32_t q_base = smem_u32(&s.q[0][0]);
    const uint32_t k_base = smem_u32(&s.k[0][0]);
    const uint32_t v_base = smem_u32(&s.v[0][0]);
    // descriptors of stage / tile bases; a k-step adds its byte offset >> 4 to
    // the start-address field (the offsets stay inside one 16 KB block)
    const uint64_t q_desc0 = sw128_desc(q_base, 16, 1024);
    const uint64_t k_desc0 = sw128_desc(k_base, 16, 1024);
    const uint64_t v_desc0 = sw128_desc(v_base, BLOCK_BYTES, 1024);
    auto issue_qk = [&](int t, int ks) {
      const uint64_t qd = q_desc0 + ((static_cast<uint32_t>(t) * TILE_BYTES) >> 4);
      const uint64_t kd = k_desc0 + ((static_cast<uint32_t>(ks) * TILE_BYTES) >> 4);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk / 4) * BLOCK_BYTES + (kk % 4) * 32) >> 4;
          mma_ss(tm_s(t), qd + off, kd + off, IDESC_QK, kk > 0 ? 1u : 0u);
        }
      }
      __syncwarp();
    };
    // half h of O_t += P_t V: keys [64h, 64h + 64)
    auto issue_pv = [&](int t, int vs, bool accumulate, int h) {
      const uint64_t vd = v_desc0 + ((static_cast<uint32_t>(vs) * TILE_BYTES) >> 4);
      if (elect_one()) {
#pragma unroll
        for (int kk = h * (BN / 32); kk < (h + 1) * (BN / 32); ++kk) {
          // A = P_t[:, 16kk:16kk+16] in TMEM (8 columns of packed bf16 pairs);
          // B = V rows 16kk.. (MN-major: 64-dim blocks BLOCK_BYTES apart, 8-row groups 1 KB apart)
          mma_ts(tm_o(t), tm_s(t) + kk * 8, vd + ((kk * 2048) >> 4), IDESC_PV,
                 (accumulate || kk > h * (BN / 32)) ? 1u : 0u);
        }
      }
      __syncwarp();
    };
    auto commit = [&](uint64_t* bar) {
      if (elect_one()) tc_commit(bar);
      __syncwarp();
    };
    ok = n_it > 0;  // (variable length: a CTA whose rows are all padding has no tile)
    if (ok && nkv0 > 0) ok = mbar_wait(&s.q_ready[0], 0);
    if (ok && nkv1 > 0) ok = mbar_wait(&s.q_ready[1], 0);
    if (ok) ok = mbar_wait(&s.k_full[0], 0);
    if (ok) {
      tc_fence_after();
      if (nkv0 > 0 && jlo0 == j_min) {
        issue_qk(0, 0);
        commit(&s.s_full[0]);
      }
      if (nkv1 > 0 && jlo1 == j_min) {
        issue_qk(1, 0);
        commit(&s.s_full[1]);
      }
      commit(&s.k_empty[0]);
    }
    // one unit's step of iteration j: O_t += P_t V_j, then S_t = Q_t K_{j+1}^T.
    // V_j and K_{j+1} are waited for only right before their first use.
    bool v_ready = false, k_ready = false;
#ifdef LA_PF_MMA_SPIN
    auto pwait = [&](uint64_t* bar, uint32_t par) { return mbar_wait_spin(bar, par); };
#else
    auto pwait = [&](uint64_t* bar, uint32_t par) { return mbar_wait(bar, par); };
#endif
    // K tile of the next streamed iteration, waited for at most once
    auto wait_next_k = [&](int it) -> bool {
      if (!k_ready) {
        if (!mbar_wait(&s.k_full[(it + 1) % KSTAGES], ((it + 1) / KSTAGES) & 1)) return false;
        k_ready = true;
      }
      return true;
    };
    // unit t over its tiles [jlo, nkv); its own tile count jj = j - jlo sets the
    // phases of its S / P barriers
    auto unit_step = [&](int t, int jlo, int nkv, int j, int it, int vs) -> bool {
      if (j + 1 == jlo) {
        // the unit starts with the next tile: its first S = Q K^T
        if (!wait_next_k(it)) return false;
        tc_fence_after();
        issue_qk(t, (it + 1) % KSTAGES);
        commit(&s.s_full[t]);
        return true;
      }
      if (j < jlo || j >= nkv) return true;
      const int jj = j - jlo;
      if (!pwait(&s.p_lo[t], jj & 1)) return false;
      if (!v_ready) {
        if (!mbar_wait(&s.v_full[vs], (it / VSTAGES) & 1)) return false;
        v_ready = true;
        if (VARLEN && (j + 1) * BN > S_b) {
          // the batch entry's last tile: its rows at or past S_b are padding
          // (any value, NaN included); zero them so that their zero weights add
          // exactly zero.  Rows stay contiguous under the swizzle.
          const int r0 = S_b - j * BN;
          uint8_t* vt = reinterpret_cast<uint8_t*>(&s.v[vs][0]);
          for (int cb = 0; cb < CB; ++cb)
            for (int idx = r0 * 8 + lane; idx < BN * 8; idx += 32)
              *reinterpret_cast<uint4*>(vt + cb * BLOCK_BYTES + idx * 16) = make_uint4(0, 0, 0, 0);
          fence_proxy_async_smem();
          __syncwarp();
        }
      }
      tc_fence_after();
      issue_pv(t, vs, jj > 0, 0);
      if (!pwait(&s.p_hi[t], jj & 1)) return false;
      tc_fence_after();
      issue_pv(t, vs, true, 1);
      if (j + 1 == nkv) {
        commit(&s.o_full[t]);
      } else {
        if (!wait_next_k(it)) return false;
        issue_qk(t, (it + 1) % KSTAGES);
        commit(&s.s_full[t]);
      }
      return true;
    };
    for (int it = 0; it < n_it && ok; ++it) {
      const int j = j_min + it;
      const int vs = it % VSTAGES;
      const bool next = it + 1 < n_it;
      v_ready = false;
      k_ready = false;
      if (nkv0 > 0) ok = unit_step(0, jlo0, nkv0, j, it, vs);
      if (ok && nkv1 > 0) ok = unit_step(1, jlo1, nkv1, j, it, vs);
      if (!ok) break;
      commit(&s.v_empty[vs]);
      if (next) commit(&s.k_empty[(it + 1) % KSTAGES]);
    }
    // every MMA this warp issued has completed before the CTA can exit
    commit(&s.mma_done);
    mbar_wait(&s.mma_done, 0);
  } else if (warp < 4) {
    setmaxnreg_dec<kRegsControl>();  // idle warps of warpgroup 0
  } else {
    // ================================================================ softmax / epilogue
    setmaxnreg_inc<kRegsSoftmax>();
    const int t = (warp - 4) >> 2;     // unit handled by this warpgroup
    const int quarter = warp & 3;      // TMEM lane quarter of this warp
    const int r = quarter * 32 + lane; // row of the Q tile = TMEM lane
    const int n_kv = t ? nkv1 : nkv0;
    const int my_pb = t ? pb1 : pb0;
    const uint32_t my_s = tm_s(t), my_o = tm_o(t);
    if (n_kv > 0) {
      const int head = t ? head1 : head0;
      const int i = my_pb * BM + r;  // query position (sequence index)
      // ---- stage Q: the raw tile arrives by TMA; rotate it in shared memory.
      // Warp-cooperative: per step a warp takes 32 / (D/4) rows, each lane one
      // bf16 pair (d, d+1) of the first half and its partner pair d + D/2, with
      // coalesced cos/sin loads; 32 lanes cover whole 128-byte rows, so the
      // swizzled accesses are free of bank conflicts.  A LLaMA cos/sin row
      // repeats its first half (the frequencies are concatenated with
      // themselves), so columns d and d + D/2 share one value and only the
      // first half is read.  The values of all the warp's rows are loaded into
      // registers at once, while the Q copy is still in flight: the table
      // reads cost one round trip.
      {
        if (p.cos != nullptr) {
          constexpr int PAIRS = D / 4;             // bf16 pairs in half a row
          constexpr int ROWS_PER_STEP = 32 / PAIRS;
          constexpr int STEPS = 32 / ROWS_PER_STEP;  // steps covering the warp's 32 rows
          uint8_t* qs = reinterpret_cast<uint8_t*>(&s.q[t][0]);
          const int wq = warp & 3;                 // warp index inside the warpgroup
          const int pr = lane % PAIRS, rsub = lane / PAIRS;
          const int d = 2 * pr;                    // first-half dim of this lane's pair
          const int d2 = d + D / 2;                // its rotation partner
          const uint32_t colb = static_cast<uint32_t>((d % 64) / 8), inb = (d % 8) * 2;
          const uint32_t colb2 = static_cast<uint32_t>((d2 % 64) / 8);
          float2 cf[STEPS], sf[STEPS];
#pragma unroll
          for (int st = 0; st < STEPS; ++st) {
            const int rr = wq * 32 + st * ROWS_PER_STEP + rsub;
            // rows past S_b are discarded (zeros, padding or the next packed
            // sequence); any of this entry's table rows serves them
            const int pos = min(my_pb * BM + rr, S_b - 1);
            const size_t trow = ((VARLEN == 2 ? static_cast<size_t>(tok0)
                                               : static_cast<size_t>(b) * p.S) + pos) * D;
            cf[st] = *reinterpret_cast<const float2*>(p.cos + trow + d);
            sf[st] = *reinterpret_cast<const float2*>(p.sin + trow + d);
          }
          if (mbar_wait(&s.q_loaded[t], 0)) {
#pragma unroll
            for (int st = 0; st < STEPS; ++st) {
              const int rr = wq * 32 + st * ROWS_PER_STEP + rsub;
              const uint32_t row = static_cast<uint32_t>(rr) * 128;
              uint32_t* p1 = reinterpret_cast<uint32_t*>(qs + (d / 64) * BLOCK_BYTES + row +
                                                         (((colb ^ (rr & 7)) << 4) | inb));
              uint32_t* p2 = reinterpret_cast<uint32_t*>(qs + (d2 / 64) * BLOCK_BYTES + row +
                                                         (((colb2 ^ (rr & 7)) << 4) | inb));
              const uint32_t xa = *p1, za = *p2;
              const float x0 = bf16lo(xa), x1 = bf16hi(xa), z0 = bf16lo(za), z1 = bf16hi(za);
              *p1 = pack_bf16x2(fmaf(x0, cf[st].x, -z0 * sf[st].x), fmaf(x1, cf[st].y, -z1 * sf[st].y));
              *p2 = pack_bf16x2(fmaf(z0, cf[st].x, x0 * sf[st].x), fmaf(z1, cf[st].y, x1 * sf[st].y));
            }
          }
          fence_proxy_async_smem();
        } else {
          mbar_wait(&s.q_loaded[t], 0);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.q_ready[t]);
      }

      const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
      const float* mrow = p.mask ? p.mask + (static_cast<size_t>(b) * p.S + i) * p.S : nullptr;
      const float c_log2 = p.scale_log2;
      const bool scale_pos = c_log2 > 0.f;
      float m_ref = -INFINITY;  // reference max (log2 units) of the exponentials
      float l_sum = 0.f;
      bool ok = true;
      const int my_jlo = t ? jlo1 : jlo0;
      for (int j = my_jlo; j < n_kv; ++j) {
        const int jj = j - my_jlo;  // this unit's tile count: barrier phases
        if (!mbar_wait(&s.s_full[t], jj & 1)) { ok = false; break; }
        tc_fence_after();
        // S in two batches: the second half is in flight while the first half's
        // max is taken
        uint32_t sr[4][32];
        tmem_ld32(my_s + lane_off, sr[0]);
        tmem_ld32(my_s + lane_off + 32, sr[1]);
        tmem_ld_wait(sr[0]);
        tmem_ld_wait(sr[1]);
        tmem_ld32(my_s + lane_off + 64, sr[2]);
        tmem_ld32(my_s + lane_off + 96, sr[3]);
        // v: raw scores (interior tiles: the scale is folded into the exponent's FMA)
        // or scaled + masked scores (tiles that touch the diagonal, the ragged end
        // or a mask, and any tile when scale <= 0)
        const int key0 = j * BN;
        const bool edge = (key0 + BN > S_b) || (p.causal && key0 + BN - 1 > my_pb * BM) ||
                          (WINDOW && key0 < my_pb * BM + BM - p.window) ||
                          (mrow != nullptr) || !scale_pos;
        float rs = 0.f;
        auto tile = [&](auto edge_c) {
          constexpr bool kEdge = decltype(edge_c)::value;
          const int lim = p.causal ? min(S_b - 1, i) : S_b - 1;  // last visible key
          const int lo = WINDOW ? i - p.window + 1 : 0;            // first visible key
          float v[BN];
          auto fill = [&](int e0) {
#pragma unroll
            for (int e = e0; e < e0 + BN / 2; ++e) {
              if (!kEdge) {
                v[e] = __uint_as_float(sr[e / 32][e % 32]);
              } else {
                const int key = key0 + e;
                float xv = __uint_as_float(sr[e / 32][e % 32]) * c_log2;
                if (mrow != nullptr && key < S_b) xv = fmaf(mrow[key], 1.4426950408889634f, xv);
                v[e] = (key <= lim && key >= lo) ? xv : -INFINITY;
              }
            }
          };
          // row max: eight independent 3-input chains, then a small tree
          float mm[8];
          fill(0);
#pragma unroll
          for (int k = 0; k < 8; ++k) mm[k] = fmaxf(v[k], v[k + 8]);
#pragma unroll
          for (int e = 16; e < BN / 2; e += 16)
#pragma unroll
            for (int k = 0; k < 8; ++k) mm[k] = fmax3f(mm[k], v[e + k], v[e + k + 8]);
          tmem_ld_wait(sr[2]);
          tmem_ld_wait(sr[3]);
          fill(BN / 2);
#pragma unroll
          for (int e = BN / 2; e < BN; e += 16)
#pragma unroll
            for (int k = 0; k < 8; ++k) mm[k] = fmax3f(mm[k], v[e + k], v[e + k + 8]);
          float mx = fmax3f(fmax3f(mm[0], mm[1], mm[2]), fmax3f(mm[3], mm[4], mm[5]),
                            fmaxf(mm[6], mm[7]));
          if (!kEdge) mx *= c_log2;
          // lazy reference: move only when the max grows by more than the threshold
          float alpha = 1.f;
          if (mx > m_ref + kRescaleThreshold || (m_ref == -INFINITY && mx != -INFINITY)) {
            alpha = (m_ref == -INFINITY) ? 0.f : ex2_approx(m_ref - mx);
            m_ref = mx;
          }
          const float nref = (m_ref == -INFINITY) ? 0.f : -m_ref;
          const float cc = kEdge ? 1.f : c_log2;
          float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
          // P in two halves (keys 0-63, 64-127): the MMA warp starts O += P V on the
          // first half while the second is being exponentiated.  The first
          // kStOverlap pairs of the second half are computed between the first
          // half's TMEM store and the wait for it, which hides the store's latency.
          uint32_t pk[2][32];
          auto exps = [&](int e0, int e1) {  // pairs of keys [e0, e1)
#pragma unroll
            for (int e = e0; e < e1; e += 2) {
              float a0, a1, p0, p1;
              ffma2(a0, a1, v[e], v[e + 1], cc, cc, nref, nref);  // exponent = v*c - m_ref
              if (!kEdge && ((e / 2) % 8) < kPolyPairsOf8) {
                exp2_poly2(p0, p1, a0, a1);
              } else {
                p0 = ex2_approx(a0);
                p1 = ex2_approx(a1);
              }
              const int k = (e / 2) % 4;
              fadd2(acc[2 * k], acc[2 * k + 1], acc[2 * k], acc[2 * k + 1], p0, p1);
              pk[e / 64][(e % 64) / 2] = pack_bf16x2(p0, p1);
            }
          };
          auto release = [&](uint64_t* bar) {
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar);
          };
          exps(0, 64);
          if (jj > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
            // O correction before any P of this tile is released (warp-collective
            // TMEM access when any row of the warp needs it); PV_{j-1} has
            // completed: its commit preceded this tile's S
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              uint32_t orr[32];
              tmem_ld32(my_o + lane_off + c * 32, orr);
              tmem_ld_wait(orr);
#pragma unroll
              for (int e = 0; e < 32; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * alpha);
              tmem_st32(my_o + lane_off + c * 32, orr);
            }
          }
          tmem_st32(my_s + lane_off, pk[0]);
          exps(64, 64 + 2 * kStOverlap);
          release(&s.p_lo[t]);
          exps(64 + 2 * kStOverlap, 128);
          tmem_st32(my_s + lane_off + 32, pk[1]);
          release(&s.p_hi[t]);
          rs = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
          l_sum = fmaf(l_sum, alpha, rs);
        };
        if (edge) tile(std::true_type{});
        else tile(std::false_type{});
      }
      // ---- epilogue: O / l -> bf16 -> out[b, i, head*D : head*D + D].  Each warp
      // writes its 32 rows into the unit's Q tile buffer (free: every MMA has
      // completed once O is final) in the same 128-byte swizzle, then one lane
      // stores them with TMA (rows past S are clipped by the tensor map) and
      // waits until the copy has read shared memory.
      if (ok && mbar_wait(&s.o_full[t], 0)) {
        tc_fence_after();
        // (variable length: rows at or past S_b are padding and come out zero;
        // select, since a padded query row may hold NaN)
        const bool pad_row = VARLEN == 1 && i >= S_b;
        const float inv = (l_sum > 0.f) ? 1.f / l_sum : 0.f;
        uint8_t* ob = reinterpret_cast<uint8_t*>(&s.q[t][0]);
        const uint32_t row = static_cast<uint32_t>(r) * 128;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t orr[32];
          tmem_ld32(my_o + lane_off + c * 32, orr);
          tmem_ld_wait(orr);
          if (pad_row)
#pragma unroll
            for (int e = 0; e < 32; ++e) orr[e] = 0u;
          const int cb = (c * 32) / 64;
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(orr[e]) * inv, __uint_as_float(orr[e + 1]) * inv);
            w.y = pack_bf16x2(__uint_as_float(orr[e + 2]) * inv, __uint_as_float(orr[e + 3]) * inv);
            w.z = pack_bf16x2(__uint_as_float(orr[e + 4]) * inv, __uint_as_float(orr[e + 5]) * inv);
            w.w = pack_bf16x2(__uint_as_float(orr[e + 6]) * inv, __uint_as_float(orr[e + 7]) * inv);
            const uint32_t chunk = static_cast<uint32_t>(((c * 32) % 64 + e) / 8);
            *reinterpret_cast<uint4*>(ob + cb * BLOCK_BYTES + row + ((chunk ^ (r & 7)) << 4)) = w;
          }
        }
        if (VARLEN != 2) {
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && my_pb * BM + quarter * 32 < p.S) {  // the box holds a row below S
#pragma unroll
            for (int cb = 0; cb < CB; ++cb)
              tma_store_4d(&tm_out, ob + cb * BLOCK_BYTES + quarter * 32 * 128, cb * 64, head,
                           my_pb * BM + quarter * 32, b);
            bulk_commit_group();
            bulk_wait_group_read0();
          }
        } else if (i < S_b) {
          // packed: the rows past S_b belong to the next sequence, so each
          // thread stores its own row (read back from the staged tile)
          __nv_bfloat16* orow = p.out + (static_cast<size_t>(tok0) + i) * (static_cast<size_t>(p.H) * D) +
                                static_cast<size_t>(head) * D;
#pragma unroll
          for (int c = 0; c < D / 8; ++c)
            *reinterpret_cast<uint4*>(orow + c * 8) = *reinterpret_cast<const uint4*>(
                ob + (c / 8) * BLOCK_BYTES + row + (((c % 8) ^ (r & 7)) << 4));
        }
        __syncwarp();
      }
    } else if (VARLEN == 1 && (t ? u1 : u0) < n_units) {
      // variable length: every row of this Q tile is padding; its output rows are zero
      const int i = my_pb * BM + r;
      if (i < p.S) {
        __nv_bfloat16* orow = p.out + (static_cast<size_t>(b) * p.S + i) * (static_cast<size_t>(p.H) * D) +
                              static_cast<size_t>(t ? head1 : head0) * D;
#pragma unroll
        for (int c = 0; c < D / 8; ++c) *reinterpret_cast<uint4*>(orow + c * 8) = make_uint4(0, 0, 0, 0);
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

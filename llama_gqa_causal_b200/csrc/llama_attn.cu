// C ABI of libllama_attn.so (declared in include/llama_attn.h): argument
// validation, TMA tensor-map encoding and kernel dispatch.  Every kernel of
// the library is compiled into this one translation unit.
#include <math.h>
#include <stdint.h>
#include <stdio.h>

#include <algorithm>
#include <cmath>
#include <mutex>

#include "llama_attn.h"

#include "common.cuh"
#include "attn_fp32.cuh"
#include "decode_bf16.cuh"
#include "gemm_sm100.cuh"
#include "prefill_sm100.cuh"
#include "rope.cuh"

namespace {

constexpr int kAbiVersion = 120;

// ---------------------------------------------------------------- host helpers
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// A tensor map is a pure function of its base address, dimensions, strides
// and box, so encoded maps are memoised: a decode loop that calls with the
// same caches every step encodes its two maps once.  Small and
// move-to-front; shared by all threads under a mutex.
struct MapKey {
  uintptr_t base;
  int rank;
  cuuint64_t dims[5];
  cuuint64_t strides[4];
  cuuint32_t box[5];
  bool operator==(const MapKey& o) const {
    if (base != o.base || rank != o.rank) return false;
    for (int i = 0; i < rank; ++i)
      if (dims[i] != o.dims[i] || box[i] != o.box[i]) return false;
    for (int i = 0; i + 1 < rank; ++i)
      if (strides[i] != o.strides[i]) return false;
    return true;
  }
};
struct MapCache {
  static constexpr int kEntries = 32;
  std::mutex mu;
  int n = 0;
  MapKey key[kEntries];
  CUtensorMap map[kEntries];
};
MapCache& map_cache() {
  static MapCache c;
  return c;
}

// bf16 tensor map with the 128-byte swizzle; dims/strides innermost first
// (strides in bytes, for dims 1..rank-1), box innermost first.
bool make_map(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
              const cuuint64_t* strides, const cuuint32_t* box) {
  MapKey k{};
  k.base = reinterpret_cast<uintptr_t>(base);
  k.rank = rank;
  for (int i = 0; i < rank; ++i) {
    k.dims[i] = dims[i];
    k.box[i] = box[i];
  }
  for (int i = 0; i + 1 < rank; ++i) k.strides[i] = strides[i];
  MapCache& c = map_cache();
  {
    std::lock_guard<std::mutex> lock(c.mu);
    for (int i = 0; i < c.n; ++i) {
      if (c.key[i] == k) {
        *m = c.map[i];
        for (int j = i; j > 0; --j) {  // move to the front
          std::swap(c.key[j], c.key[j - 1]);
          std::swap(c.map[j], c.map[j - 1]);
        }
        return true;
      }
    }
  }
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, static_cast<cuuint32_t>(rank),
                  const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  std::lock_guard<std::mutex> lock(c.mu);
  const int last = c.n < MapCache::kEntries ? c.n++ : MapCache::kEntries - 1;  // evict the oldest
  for (int j = last; j > 0; --j) {
    c.key[j] = c.key[j - 1];
    c.map[j] = c.map[j - 1];
  }
  c.key[0] = k;
  c.map[0] = *m;
  return true;
}

// Dynamic shared memory opt-in, once per (kernel, device).  Templated on the
// kernel itself so that every instantiation keeps its own flags.
template <auto kernel>
bool ensure_smem_attr(size_t bytes) {
  static bool done[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (dev >= 0 && dev < 64 && done[dev]) return true;
  cudaError_t e =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
  if (e != cudaSuccess) return false;
  if (dev >= 0 && dev < 64) done[dev] = true;
  return true;
}

int launch_status() {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    fprintf(stderr, "llama_attn: launch failed: %s\n", cudaGetErrorString(e));
    return LLAMA_ERR_CUDA;
  }
  return LLAMA_OK;
}

int check_common(int bsz, int n_heads, int n_kv_heads, int head_dim, int dtype,
                 const float* cos, const float* sin, float scale) {
  if (bsz < 1 || n_heads < 1 || n_kv_heads < 1 || head_dim < 2) return LLAMA_ERR_INVALID_ARG;
  if (n_heads % n_kv_heads != 0) return LLAMA_ERR_INVALID_ARG;
  if (head_dim % 2 != 0) return LLAMA_ERR_INVALID_ARG;
  if ((cos == nullptr) != (sin == nullptr)) return LLAMA_ERR_INVALID_ARG;
  if (!isfinite(scale)) return LLAMA_ERR_INVALID_ARG;
  if (dtype != LLAMA_DT_F32 && dtype != LLAMA_DT_BF16) return LLAMA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return LLAMA_ERR_UNSUPPORTED;
  return LLAMA_OK;
}

// ---------------------------------------------------------------- prefill dispatch
template <int D>
int prefill_bf16(const void* q, const void* k, const void* v, const float* cos, const float* sin,
                 int bsz, int H, int Hkv, int S, float scale, int causal, void* out,
                 const float* mask, void* workspace, cudaStream_t st, int window = 0,
                 const int* seq_lens = nullptr, const int* cu_seqlens = nullptr, int T = 0) {
  // packed sequences: bsz sequences of at most S tokens inside tensors of T
  // tokens, addressed as one batch entry of T rows
  const bool packed = cu_seqlens != nullptr;
  const long long rows = packed ? static_cast<long long>(T) : S;
  const long long nbat = packed ? 1 : bsz;
  const void* k_src = k;
  if (cos != nullptr) {  // rotate every K row once into the workspace
    const long long n_tok = nbat * rows;
    const long long work = n_tok * Hkv * (D / 16);
    const int threads = 256;
    const int blocks = static_cast<int>(std::min<long long>((work + threads - 1) / threads, 148LL * 16));
    la::rope_rotate_bf16_kernel<D><<<blocks, threads, 0, st>>>(
        static_cast<const __nv_bfloat16*>(k), static_cast<__nv_bfloat16*>(workspace), cos, sin,
        n_tok, Hkv);
    if (int e = launch_status()) return e;
    k_src = workspace;
  }
  CUtensorMap tq, tk, tv, to;
  const cuuint64_t qdims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H),
                               static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(nbat)};
  const cuuint64_t qstrides[3] = {static_cast<cuuint64_t>(D) * 2,
                                  static_cast<cuuint64_t>(H) * D * 2,
                                  static_cast<cuuint64_t>(rows) * H * D * 2};
  const cuuint32_t qbox[4] = {64, 1, static_cast<cuuint32_t>(la::pf::BM), 1};
  if (!make_map(&tq, q, 4, qdims, qstrides, qbox)) return LLAMA_ERR_CUDA;
  // out [b, S, H*D] has q's layout; each warp stores 32 rows
  const cuuint32_t obox[4] = {64, 1, 32, 1};
  if (!make_map(&to, out, 4, qdims, qstrides, obox)) return LLAMA_ERR_CUDA;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(Hkv),
                              static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(nbat)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * 2,
                                 static_cast<cuuint64_t>(Hkv) * D * 2,
                                 static_cast<cuuint64_t>(rows) * Hkv * D * 2};
  const cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(la::pf::BN), 1};
  if (!make_map(&tk, k_src, 4, dims, strides, box)) return LLAMA_ERR_CUDA;
  if (!make_map(&tv, v, 4, dims, strides, box)) return LLAMA_ERR_CUDA;

  la::PrefillParams p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.cos = cos;
  p.sin = sin;
  p.mask = mask;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.bsz = bsz;
  p.H = H;
  p.Hkv = Hkv;
  p.S = S;
  p.group = H / Hkv;
  p.n_pb = (S + la::pf::BM - 1) / la::pf::BM;
  p.n_kb = (S + la::pf::BN - 1) / la::pf::BN;
  p.ctas_per_kvh = (p.group * p.n_pb + la::pf::NQ - 1) / la::pf::NQ;
  {
    // bundles of (batch, K/V head) pairs whose K' and V take at most 48 MB,
    // well inside the 126 MB L2 beside the streamed q and out tiles
    const size_t kv_bytes = static_cast<size_t>(S) * D * 2 * 2;
    const size_t per = std::max<size_t>(1, (size_t{48} << 20) / kv_bytes);
    p.bkv_per_bundle = static_cast<int>(std::min<size_t>(per, static_cast<size_t>(bsz) * Hkv));
  }
  p.causal = causal ? 1 : 0;
  p.window = window;
  p.seq_lens = seq_lens;
  p.cu_seqlens = cu_seqlens;
  p.T = T;
  p.scale_log2 = scale * 1.4426950408889634f;
  const size_t smem = sizeof(la::PfSmem<D>) + 1024;
  const long long grid = static_cast<long long>(bsz) * Hkv * p.ctas_per_kvh;
  if (grid > 0x7fffffffLL) return LLAMA_ERR_INVALID_ARG;
  const unsigned g = static_cast<unsigned>(grid);
  if (window > 0) {
    if (!ensure_smem_attr<la::prefill_sm100_kernel<D, true, 0>>(smem)) return LLAMA_ERR_CUDA;
    la::prefill_sm100_kernel<D, true, 0><<<g, la::pf::THREADS, smem, st>>>(tq, tk, tv, to, p);
  } else if (seq_lens != nullptr) {
    if (!ensure_smem_attr<la::prefill_sm100_kernel<D, false, 1>>(smem)) return LLAMA_ERR_CUDA;
    la::prefill_sm100_kernel<D, false, 1><<<g, la::pf::THREADS, smem, st>>>(tq, tk, tv, to, p);
  } else if (packed) {
    if (!ensure_smem_attr<la::prefill_sm100_kernel<D, false, 2>>(smem)) return LLAMA_ERR_CUDA;
    la::prefill_sm100_kernel<D, false, 2><<<g, la::pf::THREADS, smem, st>>>(tq, tk, tv, to, p);
  } else {
    if (!ensure_smem_attr<la::prefill_sm100_kernel<D, false, 0>>(smem)) return LLAMA_ERR_CUDA;
    la::prefill_sm100_kernel<D, false, 0><<<g, la::pf::THREADS, smem, st>>>(tq, tk, tv, to, p);
  }
  return launch_status();
}

template <int D>
int attn_fp32(const float* q, const float* k, const float* v, const float* cos, const float* sin,
              const float* mask, const int* lens, float* out, int bsz, int H, int Hkv, int S,
              int L, int decode, int causal, float scale, cudaStream_t st) {
  la::Fp32Params p;
  p.q = q; p.k = k; p.v = v; p.cos = cos; p.sin = sin; p.mask = mask; p.lens = lens; p.out = out;
  p.bsz = bsz; p.H = H; p.Hkv = Hkv; p.S = S; p.L = L; p.group = H / Hkv;
  p.decode = decode; p.causal = causal ? 1 : 0; p.scale = scale;
  dim3 grid;
  if (!decode) grid = dim3((S + 31) / 32, H, bsz);
  else grid = dim3((p.group + 31) / 32, Hkv, bsz);
  la::attn_fp32_kernel<D><<<grid, 128, 0, st>>>(p);
  return launch_status();
}

int sm_count() {
  static int count[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (count[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    count[dev] = n;
  }
  return count[dev];
}

static_assert(sizeof(la::DecSmem<128>) + 1024 <= 227 * 1024, "decode shared memory exceeds 227 KB");
static_assert(sizeof(la::PfSmem<128>) + 1024 <= 227 * 1024, "prefill shared memory exceeds 227 KB");
static_assert(sizeof(la::GmSmem) + 1024 <= 227 * 1024, "projection GEMM shared memory exceeds 227 KB");

// Y = X W^T on tcgen05 (plain) or the q/k/v heads with RoPE (qkv, D = 64 / 128).
template <bool QKV, int D>
int gemm_bf16(const void* x, const void* w, int M, int N, int K, la::GemmParams p,
              cudaStream_t st) {
  CUtensorMap ta, tb;
  const cuuint64_t adims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M)};
  const cuuint64_t astr[1] = {static_cast<cuuint64_t>(K) * 2};
  const cuuint32_t abox[2] = {static_cast<cuuint32_t>(la::gm::BK), static_cast<cuuint32_t>(la::gm::BM)};
  const cuuint64_t bdims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(N)};
  const cuuint32_t bbox[2] = {static_cast<cuuint32_t>(la::gm::BK), static_cast<cuuint32_t>(la::gm::BN)};
  if (!make_map(&ta, x, 2, adims, astr, abox)) return LLAMA_ERR_CUDA;
  if (!make_map(&tb, w, 2, bdims, astr, bbox)) return LLAMA_ERR_CUDA;
  p.M = M;
  p.N = N;
  p.K = K;
  const size_t smem = sizeof(la::GmSmem) + 1024;
  if (!ensure_smem_attr<la::gemm_bf16_kernel<QKV, D>>(smem)) return LLAMA_ERR_CUDA;
  const long long tiles = static_cast<long long>((M + la::gm::BM - 1) / la::gm::BM) *
                          ((N + la::gm::BN - 1) / la::gm::BN);
  if (tiles > 0x7fffffffLL) return LLAMA_ERR_INVALID_ARG;
  const int sms = sm_count();
  if (sms <= 0) return LLAMA_ERR_CUDA;
  // persistent: one CTA per SM (198 KB of shared memory each), tiles strided by the grid
  const unsigned grid = static_cast<unsigned>(std::min<long long>(tiles, sms));
  la::gemm_bf16_kernel<QKV, D><<<grid, la::gm::THREADS, smem, st>>>(ta, tb, p);
  return launch_status();
}

template <int D>
int decode_bf16(const void* q, const void* kc, const void* vc, const int* lens, const float* cos,
                const float* sin, int bsz, int H, int Hkv, int L, float scale, void* out,
                void* workspace, cudaStream_t st, const void* k_new = nullptr,
                const void* v_new = nullptr) {
  CUtensorMap tk, tv;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(L),
                              static_cast<cuuint64_t>(bsz) * Hkv};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(L) * D * 2};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(la::dec::TR), 1};
  if (!make_map(&tk, kc, 3, dims, strides, box)) return LLAMA_ERR_CUDA;
  if (!make_map(&tv, vc, 3, dims, strides, box)) return LLAMA_ERR_CUDA;
  const int n_ctas = std::min(sm_count(), la::dec::MAX_CTAS);
  if (n_ctas <= 0) return LLAMA_ERR_CUDA;
  la::DecodeParams p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.cos = cos;
  p.sin = sin;
  p.lens = lens;
  // append mode when the new token's rows are given: the kernel writes them
  // into the caches (the public entry takes the caches as writable)
  p.k_new = static_cast<const __nv_bfloat16*>(k_new);
  p.v_new = static_cast<const __nv_bfloat16*>(v_new);
  p.k_cache = static_cast<__nv_bfloat16*>(const_cast<void*>(kc));
  p.v_cache = static_cast<__nv_bfloat16*>(const_cast<void*>(vc));
  p.ws_home = static_cast<float*>(workspace);
  p.ws_cta = p.ws_home + static_cast<size_t>(bsz) * H * la::dec::part_stride(D);
  p.ws_prefix = reinterpret_cast<int*>(p.ws_cta + static_cast<size_t>(la::dec::MAX_CTAS) * 8 *
                                                      la::dec::part_stride(D));
  p.bsz = bsz;
  p.H = H;
  p.Hkv = Hkv;
  p.L = L;
  p.group = H / Hkv;
  p.hchunks = (p.group + 7) / 8;
  p.scale_log2 = scale * 1.4426950408889634f;
  const size_t smem = sizeof(la::DecSmem<D>) + 1024;
  const int append = (k_new != nullptr) ? 1 : 0;
  // Both kernels launch as programmatic dependents of what precedes them on
  // the stream, so their blocks are scheduled while the previous grid drains.
  // Each waits on the device (griddepcontrol.wait) before it reads or writes
  // global memory.
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t scfg = {};
  scfg.gridDim = dim3(n_ctas);
  scfg.blockDim = dim3(la::dec::THREADS);
  scfg.dynamicSmemBytes = smem;
  scfg.stream = st;
  scfg.attrs = attr;
  scfg.numAttrs = 1;
  cudaError_t se;
  if (append) {
    if (!ensure_smem_attr<la::decode_bf16_kernel<D, true>>(smem)) return LLAMA_ERR_CUDA;
    se = cudaLaunchKernelEx(&scfg, la::decode_bf16_kernel<D, true>, tk, tv, p);
  } else {
    if (!ensure_smem_attr<la::decode_bf16_kernel<D, false>>(smem)) return LLAMA_ERR_CUDA;
    se = cudaLaunchKernelEx(&scfg, la::decode_bf16_kernel<D, false>, tk, tv, p);
  }
  if (se != cudaSuccess) {
    fprintf(stderr, "llama_attn: decode launch failed: %s\n", cudaGetErrorString(se));
    (void)cudaGetLastError();  // reported here, not again by a later call
    return LLAMA_ERR_CUDA;
  }
  if (int e = launch_status()) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(Hkv * p.hchunks, bsz);
  cfg.blockDim = dim3(la::dec::COMBINE_THREADS);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const float* home = p.ws_home;
  const float* ctas = p.ws_cta;
  const int* prefix = p.ws_prefix;
  __nv_bfloat16* o = static_cast<__nv_bfloat16*>(out);
  int group = p.group, hchunks = p.hchunks;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, la::decode_combine_kernel<D>, home, ctas,
                                           prefix, o, bsz, H, Hkv, group, hchunks, n_ctas);
  if (e != cudaSuccess) {
    fprintf(stderr, "llama_attn: combine launch failed: %s\n", cudaGetErrorString(e));
    (void)cudaGetLastError();  // reported here, not again by a later call
    return LLAMA_ERR_CUDA;
  }
  return launch_status();
}

// ---------------------------------------------------------------- failure-detection self-tests
// A warp waits on an mbarrier that nothing ever arrives on, with a short
// limit: the wait runs out, records the timeout in the device status word
// and the kernel returns.  No copy or MMA is in flight, so the context stays
// usable; this is the path every pipeline wait of the library takes on expiry.
__global__ void selftest_wait_timeout_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t never_armed;
  if (threadIdx.x == 0) {
    la::mbar_init(&never_armed, 1);
    la::fence_mbar_init();
  }
  __syncthreads();
  la::mbar_wait(&never_armed, 0, limit_ns);
}
__global__ void selftest_noop_kernel() {}

}  // namespace

// ---------------------------------------------------------------- decode without caller scratch
// Split-KV decode needs a scratch area for its per-split partial results.
// llama_attn_decode_noalloc takes it from this array instead of from the
// caller: it lives in the library's device image, so every GPU that loads the
// library holds it until the process exits.
namespace {
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB per GPU
}
static __device__ __align__(256) unsigned char g_decode_noalloc_scratch[kNoAllocScratchBytes];

namespace {
// Device address of the scratch array on the current device.  Host code may
// not use the array's name as a pointer (on the host it only stands for the
// symbol), so the address is looked up with that device current, on every
// call: an address kept from an earlier call would be stale once a device
// reset has reloaded the library's device code.  The lookup allocates nothing.
void* noalloc_scratch_for_current_device() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_decode_noalloc_scratch) != cudaSuccess) return nullptr;
  return p;
}
}  // namespace

extern "C" {

int llama_attn_abi_version(void) { return kAbiVersion; }

const char* llama_attn_status_string(int status) {
  switch (status) {
    case LLAMA_OK: return "ok";
    case LLAMA_ERR_INVALID_ARG: return "invalid argument";
    case LLAMA_ERR_UNSUPPORTED: return "unsupported configuration";
    case LLAMA_ERR_CUDA: return "CUDA error";
    case LLAMA_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    default: return "unknown status";
  }
}

int llama_rope_table(const long long* pos, int bsz, int seq, int head_dim, double theta,
                     double pos_scale_factor, float* cos, float* sin, void* cuda_stream) {
  if (!pos || !cos || !sin) return LLAMA_ERR_INVALID_ARG;
  if (bsz < 1 || seq < 1 || head_dim < 2 || (head_dim % 2)) return LLAMA_ERR_INVALID_ARG;
  if (!(theta > 0.0) || !(pos_scale_factor > 0.0)) return LLAMA_ERR_INVALID_ARG;
  const long long n = static_cast<long long>(bsz) * seq;
  // a multiple of head_dim / 2 threads per block (one frequency index each)
  const int half = head_dim / 2;
  const int threads = half >= 256 ? half : (256 / half) * half;
  const long long rows_per_block = threads / half;
  const int blocks =
      static_cast<int>(std::min<long long>((n + rows_per_block - 1) / rows_per_block, 148LL * 32));
  if (threads > 1024) return LLAMA_ERR_UNSUPPORTED;
  // the inverse frequencies theta^(-2i/D), i < D/2, formed once here in
  // double rather than by every thread of the kernel
  la::RopeFreqs freqs{};
  if (half <= la::kRopeHostFreqs)
    for (int i = 0; i < half; ++i)
      freqs.inv[i] = std::exp(-(2.0 * i / head_dim) * std::log(theta));
  // launched as a programmatic dependent of the preceding grid: the launch
  // overlaps that grid's drain, and the kernel waits for it on the device
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(blocks);
  cfg.blockDim = dim3(threads);
  cfg.stream = as_stream(cuda_stream);
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, la::rope_table_kernel, pos, n, head_dim, theta,
                                           pos_scale_factor, cos, sin, freqs);
  if (e != cudaSuccess) {
    fprintf(stderr, "llama_attn: rope table launch failed: %s\n", cudaGetErrorString(e));
    (void)cudaGetLastError();  // reported here, not again by a later call
    return LLAMA_ERR_CUDA;
  }
  return launch_status();
}

int llama_rope_table_ntk(const long long* pos, int bsz, int seq, int head_dim, double theta,
                         double alpha, float* cos, float* sin, void* cuda_stream) {
  if (head_dim < 4 || !(alpha > 0.0)) return LLAMA_ERR_INVALID_ARG;
  // the NTK-aware base theta * alpha^(D / (D - 2)), then the plain table
  const double base = theta * std::pow(alpha, static_cast<double>(head_dim) / (head_dim - 2));
  if (!std::isfinite(base)) return LLAMA_ERR_INVALID_ARG;
  return llama_rope_table(pos, bsz, seq, head_dim, base, 1.0, cos, sin, cuda_stream);
}

int llama_attn_qkv_rope(const void* x, const void* w_qkv, const float* cos, const float* sin,
                        int tokens, int hidden, int n_heads, int n_kv_heads, int head_dim,
                        void* q, void* k, void* v, int dtype, void* cuda_stream) {
  if (!x || !w_qkv || !q || !k || !v) return LLAMA_ERR_INVALID_ARG;
  if (tokens < 1 || hidden < 1 || (hidden % 8)) return LLAMA_ERR_INVALID_ARG;
  if (int e = check_common(1, n_heads, n_kv_heads, head_dim, dtype, cos, sin, 1.0f)) return e;
  if (!aligned16(x) || !aligned16(w_qkv) || !aligned16(q) || !aligned16(k) || !aligned16(v) ||
      !aligned16(cos) || !aligned16(sin))
    return LLAMA_ERR_INVALID_ARG;
  if (dtype != LLAMA_DT_BF16) return LLAMA_ERR_UNSUPPORTED;
  const long long n_out = static_cast<long long>(n_heads + 2 * n_kv_heads) * head_dim;
  if (n_out > 0x7fffffffLL) return LLAMA_ERR_INVALID_ARG;
  la::GemmParams p{};
  p.q = static_cast<__nv_bfloat16*>(q);
  p.k = static_cast<__nv_bfloat16*>(k);
  p.v = static_cast<__nv_bfloat16*>(v);
  p.cos = cos;
  p.sin = sin;
  p.H = n_heads;
  p.Hkv = n_kv_heads;
  cudaStream_t st = as_stream(cuda_stream);
  if (head_dim == 128)
    return gemm_bf16<true, 128>(x, w_qkv, tokens, static_cast<int>(n_out), hidden, p, st);
  return gemm_bf16<true, 64>(x, w_qkv, tokens, static_cast<int>(n_out), hidden, p, st);
}

int llama_attn_out_proj(const void* attn, const void* w_o, int tokens, int in_dim, int out_dim,
                        void* y, int dtype, void* cuda_stream) {
  if (!attn || !w_o || !y) return LLAMA_ERR_INVALID_ARG;
  if (tokens < 1 || in_dim < 1 || out_dim < 1 || (in_dim % 8) || (out_dim % 8))
    return LLAMA_ERR_INVALID_ARG;
  if (dtype != LLAMA_DT_BF16 && dtype != LLAMA_DT_F32) return LLAMA_ERR_INVALID_ARG;
  if (!aligned16(attn) || !aligned16(w_o) || !aligned16(y)) return LLAMA_ERR_INVALID_ARG;
  if (dtype != LLAMA_DT_BF16) return LLAMA_ERR_UNSUPPORTED;
  la::GemmParams p{};
  p.y = static_cast<__nv_bfloat16*>(y);
  return gemm_bf16<false, 128>(attn, w_o, tokens, out_dim, in_dim, p, as_stream(cuda_stream));
}

size_t llama_attn_prefill_workspace_bytes(int bsz, int n_heads, int n_kv_heads, int seq,
                                          int head_dim, int dtype, int has_rope) {
  (void)n_heads;
  if (dtype != LLAMA_DT_BF16 || !has_rope || bsz < 1 || n_kv_heads < 1 || seq < 1 || head_dim < 1)
    return 0;
  return static_cast<size_t>(bsz) * seq * n_kv_heads * head_dim * 2;  // rotated K, bf16
}

int llama_attn_prefill(const void* q, const void* k, const void* v, const float* cos,
                       const float* sin, int bsz, int n_heads, int n_kv_heads, int seq,
                       int head_dim, float scale, int causal, void* out,
                       const float* add_mask, int dtype, void* workspace,
                       size_t workspace_bytes, void* cuda_stream) {
  if (!q || !k || !v || !out) return LLAMA_ERR_INVALID_ARG;
  if (seq < 1) return LLAMA_ERR_INVALID_ARG;
  if (int e = check_common(bsz, n_heads, n_kv_heads, head_dim, dtype, cos, sin, scale)) return e;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(cos) ||
      !aligned16(sin) || !aligned16(add_mask) || !aligned16(workspace))
    return LLAMA_ERR_INVALID_ARG;
  const size_t need = llama_attn_prefill_workspace_bytes(bsz, n_heads, n_kv_heads, seq, head_dim,
                                                         dtype, cos != nullptr);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return LLAMA_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(cuda_stream);
  if (dtype == LLAMA_DT_BF16) {
    if (head_dim == 128)
      return prefill_bf16<128>(q, k, v, cos, sin, bsz, n_heads, n_kv_heads, seq, scale, causal,
                               out, add_mask, workspace, st);
    return prefill_bf16<64>(q, k, v, cos, sin, bsz, n_heads, n_kv_heads, seq, scale, causal, out,
                            add_mask, workspace, st);
  }
  const float* qf = static_cast<const float*>(q);
  const float* kf = static_cast<const float*>(k);
  const float* vf = static_cast<const float*>(v);
  float* of = static_cast<float*>(out);
  if (head_dim == 128)
    return attn_fp32<128>(qf, kf, vf, cos, sin, add_mask, nullptr, of, bsz, n_heads, n_kv_heads,
                          seq, seq, 0, causal, scale, st);
  return attn_fp32<64>(qf, kf, vf, cos, sin, add_mask, nullptr, of, bsz, n_heads, n_kv_heads, seq,
                       seq, 0, causal, scale, st);
}

int llama_attn_prefill_window(const void* q, const void* k, const void* v, const float* cos,
                              const float* sin, int bsz, int n_heads, int n_kv_heads, int seq,
                              int head_dim, float scale, int window, void* out, int dtype,
                              void* workspace, size_t workspace_bytes, void* cuda_stream) {
  if (!q || !k || !v || !out) return LLAMA_ERR_INVALID_ARG;
  if (seq < 1 || window < 1) return LLAMA_ERR_INVALID_ARG;
  if (int e = check_common(bsz, n_heads, n_kv_heads, head_dim, dtype, cos, sin, scale)) return e;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(cos) ||
      !aligned16(sin) || !aligned16(workspace))
    return LLAMA_ERR_INVALID_ARG;
  if (dtype != LLAMA_DT_BF16) return LLAMA_ERR_UNSUPPORTED;
  const size_t need = llama_attn_prefill_workspace_bytes(bsz, n_heads, n_kv_heads, seq, head_dim,
                                                         dtype, cos != nullptr);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return LLAMA_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(cuda_stream);
  // a window of seq keys or more is plain causal attention
  const int w = window >= seq ? 0 : window;
  if (head_dim == 128)
    return prefill_bf16<128>(q, k, v, cos, sin, bsz, n_heads, n_kv_heads, seq, scale, 1, out,
                             nullptr, workspace, st, w);
  return prefill_bf16<64>(q, k, v, cos, sin, bsz, n_heads, n_kv_heads, seq, scale, 1, out, nullptr,
                          workspace, st, w);
}

int llama_attn_prefill_varlen(const void* q, const void* k, const void* v, const float* cos,
                              const float* sin, const int* seq_lens, int bsz, int n_heads,
                              int n_kv_heads, int seq, int head_dim, float scale, int causal,
                              void* out, int dtype, void* workspace, size_t workspace_bytes,
                              void* cuda_stream) {
  if (!q || !k || !v || !out || !seq_lens) return LLAMA_ERR_INVALID_ARG;
  if (seq < 1) return LLAMA_ERR_INVALID_ARG;
  if (int e = check_common(bsz, n_heads, n_kv_heads, head_dim, dtype, cos, sin, scale)) return e;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(cos) ||
      !aligned16(sin) || !aligned16(workspace) || (reinterpret_cast<uintptr_t>(seq_lens) & 3u))
    return LLAMA_ERR_INVALID_ARG;
  if (dtype != LLAMA_DT_BF16) return LLAMA_ERR_UNSUPPORTED;
  const size_t need = llama_attn_prefill_workspace_bytes(bsz, n_heads, n_kv_heads, seq, head_dim,
                                                         dtype, cos != nullptr);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return LLAMA_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(cuda_stream);
  if (head_dim == 128)
    return prefill_bf16<128>(q, k, v, cos, sin, bsz, n_heads, n_kv_heads, seq, scale, causal, out,
                             nullptr, workspace, st, 0, seq_lens);
  return prefill_bf16<64>(q, k, v, cos, sin, bsz, n_heads, n_kv_heads, seq, scale, causal, out,
                          nullptr, workspace, st, 0, seq_lens);
}

int llama_attn_prefill_packed(const void* q, const void* k, const void* v, const float* cos,
                              const float* sin, const int* cu_seqlens, int n_seqs,
                              int total_tokens, int max_seqlen, int n_heads, int n_kv_heads,
                              int head_dim, float scale, int causal, void* out, int dtype,
                              void* workspace, size_t workspace_bytes, void* cuda_stream) {
  if (!q || !k || !v || !out || !cu_seqlens) return LLAMA_ERR_INVALID_ARG;
  if (total_tokens < 1 || max_seqlen < 1) return LLAMA_ERR_INVALID_ARG;
  if (int e = check_common(n_seqs, n_heads, n_kv_heads, head_dim, dtype, cos, sin, scale)) return e;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(cos) ||
      !aligned16(sin) || !aligned16(workspace) || (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u))
    return LLAMA_ERR_INVALID_ARG;
  if (dtype != LLAMA_DT_BF16) return LLAMA_ERR_UNSUPPORTED;
  const size_t need = llama_attn_prefill_workspace_bytes(1, n_heads, n_kv_heads, total_tokens,
                                                         head_dim, dtype, cos != nullptr);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return LLAMA_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(cuda_stream);
  if (head_dim == 128)
    return prefill_bf16<128>(q, k, v, cos, sin, n_seqs, n_heads, n_kv_heads, max_seqlen, scale,
                             causal, out, nullptr, workspace, st, 0, nullptr, cu_seqlens,
                             total_tokens);
  return prefill_bf16<64>(q, k, v, cos, sin, n_seqs, n_heads, n_kv_heads, max_seqlen, scale, causal,
                          out, nullptr, workspace, st, 0, nullptr, cu_seqlens, total_tokens);
}

size_t llama_attn_decode_workspace_bytes(int bsz, int n_heads, int max_cache_len, int head_dim) {
  if (bsz < 1 || n_heads < 1 || max_cache_len < 1 || head_dim < 1) return 0;
  // one partial per (batch, head) plus one per (CTA, head of an 8-head
  // chunk), then the chunk prefix over the batch
  const size_t rows = static_cast<size_t>(bsz) * n_heads + static_cast<size_t>(la::dec::MAX_CTAS) * 8;
  return rows * la::dec::part_stride(head_dim) * sizeof(float) + la::dec::ws_prefix_bytes(bsz);
}

int llama_attn_decode(const void* q, const void* k_cache, const void* v_cache,
                      const int* cache_lens, const float* cos, const float* sin, int bsz,
                      int n_heads, int n_kv_heads, int max_cache_len, int head_dim,
                      float scale, void* out, void* workspace, size_t workspace_bytes,
                      int dtype, void* cuda_stream) {
  if (!q || !k_cache || !v_cache || !cache_lens || !out) return LLAMA_ERR_INVALID_ARG;
  if (max_cache_len < 1) return LLAMA_ERR_INVALID_ARG;
  if (int e = check_common(bsz, n_heads, n_kv_heads, head_dim, dtype, cos, sin, scale)) return e;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
      !aligned16(cos) || !aligned16(sin) || !aligned16(workspace) ||
      (reinterpret_cast<uintptr_t>(cache_lens) & 3u))
    return LLAMA_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(cuda_stream);
  if (dtype == LLAMA_DT_BF16) {
    if (bsz > la::dec::MAX_BATCH) return LLAMA_ERR_UNSUPPORTED;
    const size_t need = llama_attn_decode_workspace_bytes(bsz, n_heads, max_cache_len, head_dim);
    if (workspace == nullptr || workspace_bytes < need) return LLAMA_ERR_INVALID_ARG;
    if (head_dim == 128)
      return decode_bf16<128>(q, k_cache, v_cache, cache_lens, cos, sin, bsz, n_heads, n_kv_heads,
                              max_cache_len, scale, out, workspace, st);
    return decode_bf16<64>(q, k_cache, v_cache, cache_lens, cos, sin, bsz, n_heads, n_kv_heads,
                           max_cache_len, scale, out, workspace, st);
  }
  const float* qf = static_cast<const float*>(q);
  if (head_dim == 128)
    return attn_fp32<128>(qf, static_cast<const float*>(k_cache),
                          static_cast<const float*>(v_cache), cos, sin, nullptr, cache_lens,
                          static_cast<float*>(out), bsz, n_heads, n_kv_heads, 1, max_cache_len, 1,
                          0, scale, st);
  return attn_fp32<64>(qf, static_cast<const float*>(k_cache), static_cast<const float*>(v_cache),
                       cos, sin, nullptr, cache_lens, static_cast<float*>(out), bsz, n_heads,
                       n_kv_heads, 1, max_cache_len, 1, 0, scale, st);
}

int llama_attn_decode_append(const void* q, const void* k_new, const void* v_new,
                             void* k_cache, void* v_cache, const int* cache_lens,
                             const float* cos, const float* sin, int bsz, int n_heads,
                             int n_kv_heads, int max_cache_len, int head_dim, float scale,
                             void* out, void* workspace, size_t workspace_bytes, int dtype,
                             void* cuda_stream) {
  if (!q || !k_new || !v_new || !k_cache || !v_cache || !cache_lens || !out)
    return LLAMA_ERR_INVALID_ARG;
  if (max_cache_len < 1) return LLAMA_ERR_INVALID_ARG;
  if (int e = check_common(bsz, n_heads, n_kv_heads, head_dim, dtype, cos, sin, scale)) return e;
  if (!aligned16(q) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) ||
      !aligned16(v_cache) || !aligned16(out) || !aligned16(cos) || !aligned16(sin) ||
      !aligned16(workspace) || (reinterpret_cast<uintptr_t>(cache_lens) & 3u))
    return LLAMA_ERR_INVALID_ARG;
  if (dtype != LLAMA_DT_BF16) return LLAMA_ERR_UNSUPPORTED;
  if (bsz > la::dec::MAX_BATCH) return LLAMA_ERR_UNSUPPORTED;
  const size_t need = llama_attn_decode_workspace_bytes(bsz, n_heads, max_cache_len, head_dim);
  if (workspace == nullptr || workspace_bytes < need) return LLAMA_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(cuda_stream);
  if (head_dim == 128)
    return decode_bf16<128>(q, k_cache, v_cache, cache_lens, cos, sin, bsz, n_heads, n_kv_heads,
                            max_cache_len, scale, out, workspace, st, k_new, v_new);
  return decode_bf16<64>(q, k_cache, v_cache, cache_lens, cos, sin, bsz, n_heads, n_kv_heads,
                         max_cache_len, scale, out, workspace, st, k_new, v_new);
}


int llama_attn_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                              const int* cache_lens, const float* cos, const float* sin, int bsz,
                              int n_heads, int n_kv_heads, int max_cache_len, int head_dim,
                              float scale, void* out, int dtype, void* cuda_stream) {
  if (dtype == LLAMA_DT_BF16) {
    // reject requests the static scratch cannot hold before touching the device
    if (bsz >= 1 && n_heads >= 1 && max_cache_len >= 1 && head_dim >= 1 &&
        llama_attn_decode_workspace_bytes(bsz, n_heads, max_cache_len, head_dim) >
            kNoAllocScratchBytes) {
      fprintf(stderr,
              "llama_attn_decode_noalloc: %zu bytes of scratch needed, the static limit is %zu; "
              "use llama_attn_decode with a caller workspace\n",
              llama_attn_decode_workspace_bytes(bsz, n_heads, max_cache_len, head_dim),
              kNoAllocScratchBytes);
      return LLAMA_ERR_INVALID_ARG;
    }
  }
  void* scratch = nullptr;
  if (dtype == LLAMA_DT_BF16 && q && k_cache && v_cache && cache_lens && out) {
    scratch = noalloc_scratch_for_current_device();
    if (scratch == nullptr) return LLAMA_ERR_CUDA;
  }
  return llama_attn_decode(q, k_cache, v_cache, cache_lens, cos, sin, bsz, n_heads, n_kv_heads,
                           max_cache_len, head_dim, scale, out, scratch,
                           scratch ? kNoAllocScratchBytes : 0, dtype, cuda_stream);
}

int llama_attn_selftest_wait_timeout(unsigned int limit_us, void* cuda_stream) {
  if (limit_us < 1 || limit_us > 1000000u) return LLAMA_ERR_INVALID_ARG;
  selftest_wait_timeout_kernel<<<1, 32, 0, as_stream(cuda_stream)>>>(
      static_cast<unsigned long long>(limit_us) * 1000ull);
  return launch_status();
}

int llama_attn_selftest_launch_error(void* cuda_stream) {
  // 2048 threads per block exceeds the 1024 every CUDA device allows: the
  // runtime refuses the launch on the host, before anything reaches the GPU
  selftest_noop_kernel<<<1, 2048, 0, as_stream(cuda_stream)>>>();
  return launch_status();
}

int llama_attn_device_status(void* cuda_stream) {
  if (cudaStreamSynchronize(as_stream(cuda_stream)) != cudaSuccess) return LLAMA_ERR_CUDA;
  unsigned int word = 0;
  if (cudaMemcpyFromSymbol(&word, la::g_device_status, sizeof(word)) != cudaSuccess)
    return LLAMA_ERR_CUDA;
  if (word != 0) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(la::g_device_status, &zero, sizeof(zero)) != cudaSuccess)
      return LLAMA_ERR_CUDA;
    return LLAMA_ERR_DEVICE_TIMEOUT;
  }
  return LLAMA_OK;
}

}  // extern "C"

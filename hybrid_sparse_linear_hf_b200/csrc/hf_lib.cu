// C ABI of the hybrid attention chunk step (declared in include/hf.h).
//
// Host side: argument validation (before any launch), TMA tensor-map encoding, grid
// sizing and kernel dispatch on (d, block). The whole library is this one translation
// unit; the kernels live in the included headers.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "hf.h"
#include "hf_absorb.cuh"
#include "hf_attn.cuh"
#include "hf_ptx.cuh"
#include "hf_select.cuh"

namespace {


constexpr unsigned long long kDefaultTimeoutNs = 1000000000ull;  // 1 s per wait
// CTAs the absorption spreads a call over (one per SM of a B200). A constant, so the
// workspace size is a pure function of the shapes.
constexpr int kAbsorbTargetCtas = 148;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

std::mutex g_mu;
EncodeTiledFn g_encode = nullptr;

struct Injection {
  int kernel_id = 0;
  int count = 0;
  unsigned long long timeout_ns = kDefaultTimeoutNs;
};
Injection g_inject;

// Returns (inject flag, timeout) for one launch of `kernel_id`.
void take_injection(int kernel_id, int* inject, unsigned long long* timeout_ns) {
  std::lock_guard<std::mutex> lk(g_mu);
  *inject = 0;
  *timeout_ns = kDefaultTimeoutNs;
  if (g_inject.kernel_id == kernel_id && g_inject.count > 0) {
    *inject = 1;
    *timeout_ns = g_inject.timeout_ns;
    if (--g_inject.count == 0) g_inject.kernel_id = 0;
  }
}

EncodeTiledFn encoder() {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  }
  return g_encode;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool supported_d(int d) { return d == 64 || d == 128; }
bool supported_block(int b) { return b == 32 || b == 64 || b == 128; }
int ceil_div(long long a, long long b) { return static_cast<int>((a + b - 1) / b); }
size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// 3-D bf16 tensor map over [BH][rows][d] with a (64 x box_rows x 1) box, 128-byte swizzle.
hf_status make_map(CUtensorMap* m, const void* base, int d, long long rows, long long bh, int box_rows) {
  EncodeTiledFn enc = encoder();
  if (!enc) return HF_ERR_CUDA;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(bh)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(rows) * d * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? HF_OK : HF_ERR_CUDA;
}

// Kernels this library instance has launched (reported by hf_launch_count).
std::atomic<unsigned long long> g_launches{0};

// Status of the launch just issued; a successful one is counted.
hf_status launch_status() {
  if (cudaGetLastError() != cudaSuccess) return HF_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return HF_OK;
}

// Launches `kernel` with programmatic stream serialisation: it may be scheduled before the
// previous kernel of the stream has finished (once every CTA of that one has started);
// each kernel of the library waits for its predecessor (griddep_wait) before it reads
// anything that one may have written. The launch is counted on success.
template <typename... KArgs, typename... Args>
hf_status launch_pdl(void (*kernel)(KArgs...), long long grid, int block, size_t smem, cudaStream_t st,
                     Args... args) {
  if (grid < 1 || grid > 0x7fffffffLL) return HF_ERR_UNSUPPORTED;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(static_cast<unsigned>(block));
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...) != cudaSuccess) {
    cudaGetLastError();
    return HF_ERR_CUDA;
  }
  return launch_status();
}

// Checks of an hf_rope for a step with Nq queries, a window of Nk keys and blocks of
// `block` tokens: the chunk must lie inside the window's frames.
bool rope_ok(const hf_rope* rope, int d, int Nq, int Nk, int block) {
  if (!rope) return false;
  if (rope->d_t < 0 || (rope->d_t & 1) || rope->d_t > d || rope->d_t > 64) return false;
  if (rope->tokens_per_frame < block || rope->cap < 0 || rope->cap > 63) return false;
  if (!(rope->base > 1.0f) || std::isinf(rope->base)) return false;
  const int W = ceil_div(Nk, rope->tokens_per_frame);
  return rope->q_frame0 >= 0 && static_cast<long long>(rope->q_frame0) + ceil_div(Nq, rope->tokens_per_frame) <= W;
}

// Arguments of the block pooling of Q (and K unless nKB == 0); with a rope, the means of
// the turned tokens.
hf::PoolArgs pool_args(const hf_bf16* Q, const hf_bf16* K, int Nq, int Nk, int block, int nQB, int nKB, float* Qp,
                       float* Kp, int T, float* Kpart, const hf_rope* rope) {
  hf::PoolArgs a;
  a.Q = reinterpret_cast<const __nv_bfloat16*>(Q);
  a.K = reinterpret_cast<const __nv_bfloat16*>(K);
  a.Nq = Nq;
  a.Nk = Nk;
  a.block = block;
  a.nQB = nQB;
  a.nKB = nKB;
  a.Qp = Qp;
  a.Kp = Kp;
  a.T = T;
  a.Kpart = Kpart;
  a.q_frame0 = a.n_frames = a.rope_cap = a.rope_dt = 0;
  a.rope_log2base = 0.f;
  a.k_transposed = 0;
  if (rope) {
    a.T = rope->tokens_per_frame;
    a.q_frame0 = rope->q_frame0;
    a.n_frames = ceil_div(Nk, rope->tokens_per_frame);
    a.rope_cap = rope->cap;
    a.rope_dt = rope->d_t;
    a.rope_log2base = std::log2(rope->base);
  }
  return a;
}

// Block pooling (the means of Q's and K's blocks into the workspace; the key means
// transposed with `k_transposed`).
template <int D, bool kParts, bool kRope = false>
hf_status launch_pool(const hf_bf16* Q, const hf_bf16* K, int BH, int Nq, int Nk, int block, int nQB, int nKB,
                      float* Qp, float* Kp, int T, float* Kpart, cudaStream_t st, const hf_rope* rope = nullptr,
                      bool k_transposed = false) {
  hf::PoolArgs a = pool_args(Q, K, Nq, Nk, block, nQB, nKB, Qp, Kp, T, Kpart, kRope ? rope : nullptr);
  a.k_transposed = k_transposed ? 1 : 0;
  return launch_pdl(hf::pool_blocks_kernel<D, kParts, kRope>, static_cast<long long>(BH) * (nQB + nKB),
                    hf::kPoolThreads, 0, st, a);
}

// ---------------------------------------------------------------- select
size_t select_ws_bytes(int B, int H, int Nq, int Nk, int d, int block) {
  const long long bh = static_cast<long long>(B) * H;
  return align256(static_cast<size_t>(bh) * ceil_div(Nq, block) * d * 4) +
         align256(static_cast<size_t>(bh) * ceil_div(Nk, block) * d * 4);
}

// The selection's grids fit the launch limit (a pooling CTA per block).
bool select_grid_ok(long long BH, int Nq, int nKB, int block) {
  return BH * (ceil_div(Nq, block) + nKB) <= 0x7fffffffLL;
}

// Whether the scores come from the staged kernel (the pooling then writes the key means
// transposed).
template <int D>
bool staged_scores(int nKB) {
  return static_cast<long long>(nKB) * D * 4 <= hf::kStagedKBytes;
}

// Scores and top-r from the pooled means in the workspace: the staged kernel on
// transposed key means (`transposed`), else the plain kernel on row-major means.
template <int D>
hf_status launch_score(const float* Qp, const float* Kp, int BH, int nQB, int nKB, int r, int32_t* idx,
                       float* scores, cudaStream_t st, bool transposed) {
  const long long groups = (nQB + hf::kSelQB - 1) / hf::kSelQB;
  if (transposed) {
    const size_t smem = static_cast<size_t>(nKB) * D * 4 + static_cast<size_t>(nKB) * hf::kSelQB * sizeof(float);
    if (cudaFuncSetAttribute(hf::score_select_staged_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return HF_ERR_CUDA;
    int inject = 0;
    unsigned long long timeout_ns = kDefaultTimeoutNs;
    take_injection(1, &inject, &timeout_ns);
    return launch_pdl(hf::score_select_staged_kernel<D>, BH * groups, hf::kSelectThreads, smem, st, Qp, Kp, nQB, nKB,
                      r, idx, scores, timeout_ns, inject);
  }
  // the opt-in covers static + dynamic shared memory above the 48 KB default; set on
  // every launch so that no size of nKB depends on it having been set before
  const size_t smem = static_cast<size_t>(nKB) * hf::kSelQB * sizeof(float);
  if (cudaFuncSetAttribute(hf::score_select_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return HF_ERR_CUDA;
  return launch_pdl(hf::score_select_kernel<D>, BH * groups, hf::kSelectThreads, smem, st, Qp, Kp, nQB, nKB, r, idx,
                    scores);
}

template <int D>
hf_status launch_select(const hf_bf16* Q, const hf_bf16* K, int BH, int Nq, int Nk, int block, int r,
                        int32_t* idx, float* scores, void* ws, cudaStream_t st, const hf_rope* rope = nullptr) {
  const int nQB = ceil_div(Nq, block), nKB = ceil_div(Nk, block);
  float* Qp = static_cast<float*>(ws);
  float* Kp = reinterpret_cast<float*>(static_cast<char*>(ws) + align256(static_cast<size_t>(BH) * nQB * D * 4));
  const bool staged = staged_scores<D>(nKB);
  const hf_status rc = rope ? launch_pool<D, false, true>(Q, K, BH, Nq, Nk, block, nQB, nKB, Qp, Kp, 0, nullptr, st,
                                                            rope, staged)
                            : launch_pool<D, false>(Q, K, BH, Nq, Nk, block, nQB, nKB, Qp, Kp, 0, nullptr, st,
                                                    nullptr, staged);
  if (rc != HF_OK) return HF_ERR_CUDA;
  return launch_score<D>(Qp, Kp, BH, nQB, nKB, r, idx, scores, st, staged);
}

// selection over the pooled-key cache: Q pooled as above (no key blocks), key blocks from
// the granule sums
// (with `push`: the push's granule sums are computed by the CTAs after the Q pooling's,
// in the same launch; kp is then the window after the push)
template <int D>
hf_status launch_select_cached(const hf_bf16* Q, const hf_kpool* kp, int BH, int Nq, int Nk, int block, int r,
                               int32_t* idx, float* scores, void* ws, cudaStream_t st,
                               const hf::PushArgs* push = nullptr, long long push_ctas = 0) {
  const int nQB = ceil_div(Nq, block), nKB = ceil_div(Nk, block);
  float* Qp = static_cast<float*>(ws);
  float* Kp = reinterpret_cast<float*>(static_cast<char*>(ws) + align256(static_cast<size_t>(BH) * nQB * D * 4));
  if (push) {
    const hf::PoolArgs a = pool_args(Q, nullptr, Nq, 0, block, nQB, 0, Qp, Kp, 0, nullptr, nullptr);
    const long long q_ctas = static_cast<long long>(BH) * nQB;
    if (launch_pdl(hf::pool_q_push_kernel<D>, q_ctas + push_ctas, hf::kPoolThreads, 0, st, a, *push,
                   static_cast<int>(q_ctas)) != HF_OK)
      return HF_ERR_CUDA;
  } else if (launch_pool<D, false>(Q, nullptr, BH, Nq, 0, block, nQB, 0, Qp, Kp, 0, nullptr, st) != HF_OK) {
    return HF_ERR_CUDA;
  }
  constexpr int kWarpsPerCta = hf::kPoolThreads / 32;
  const bool staged = staged_scores<D>(nKB);
  const float* sums = static_cast<const float*>(kp->sums);
  const hf_status rc =
      staged ? launch_pdl(hf::kpool_blocks_kernel<D, true>,
                          static_cast<long long>(BH) * ((nKB + kWarpsPerCta - 1) / kWarpsPerCta), hf::kPoolThreads, 0,
                          st, sums, kp->capacity, kp->head, kp->n_gran, kp->granule, block, nKB, BH, Kp)
             : launch_pdl(hf::kpool_blocks_kernel<D, false>,
                          (static_cast<long long>(BH) * nKB + kWarpsPerCta - 1) / kWarpsPerCta, hf::kPoolThreads, 0,
                          st, sums, kp->capacity, kp->head, kp->n_gran, kp->granule, block, nKB, BH, Kp);
  if (rc != HF_OK) return HF_ERR_CUDA;
  return launch_score<D>(Qp, Kp, BH, nQB, nKB, r, idx, scores, st, staged);
}

// ---------------------------------------------------------------- two-stage select
// Workspace: pooled Q, pooled K, the key blocks' frame parts and the frame means (fp32);
// W <= nKB because tokens_per_frame >= block.
size_t select2_ws_bytes(int B, int H, int Nq, int Nk, int d, int block) {
  const long long bh = static_cast<long long>(B) * H;
  const size_t nKB = ceil_div(Nk, block);
  return align256(static_cast<size_t>(bh) * ceil_div(Nq, block) * d * 4) + align256(bh * nKB * d * 4) +
         align256(bh * nKB * 2 * d * 4) + align256(bh * nKB * d * 4);
}

template <int D>
hf_status launch_select2(const hf_bf16* Q, const hf_bf16* K, int BH, int Nq, int Nk, int block, int r, int T, int nf,
                         int32_t* idx, int32_t* frames, float* scores, void* ws, cudaStream_t st) {
  const int nQB = ceil_div(Nq, block), nKB = ceil_div(Nk, block), W = ceil_div(Nk, T);
  char* base = static_cast<char*>(ws);
  float* Qp = reinterpret_cast<float*>(base);
  base += align256(static_cast<size_t>(BH) * nQB * D * 4);
  float* Kp = reinterpret_cast<float*>(base);
  base += align256(static_cast<size_t>(BH) * nKB * D * 4);
  float* Kpart = reinterpret_cast<float*>(base);
  base += align256(static_cast<size_t>(BH) * nKB * 2 * D * 4);
  float* Kf = reinterpret_cast<float*>(base);
  if (launch_pool<D, true>(Q, K, BH, Nq, Nk, block, nQB, nKB, Qp, Kp, T, Kpart, st) != HF_OK) return HF_ERR_CUDA;
  if (launch_pdl(hf::pool_frames_kernel<D>, static_cast<long long>(BH) * W, D, 0, st, static_cast<const float*>(Kpart),
                 Nk, block, T, nKB, W, Kf) != HF_OK)
    return HF_ERR_CUDA;
  const size_t smem = static_cast<size_t>(hf::kSelQB) * (nKB + W) * (sizeof(float) + 1);
  if (cudaFuncSetAttribute(hf::score_select2_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return HF_ERR_CUDA;
  const long long groups = (nQB + hf::kSelQB - 1) / hf::kSelQB;
  return launch_pdl(hf::score_select2_kernel<D>, static_cast<long long>(BH) * groups, hf::kSelectThreads, smem, st,
                    static_cast<const float*>(Qp), static_cast<const float*>(Kp), static_cast<const float*>(Kf), nQB,
                    nKB, W, Nk, block, T, r, nf, idx, frames, scores);
}

// ---------------------------------------------------------------- absorb
struct AbsorbPlan {
  int tiles_per_split, nsplit;
};

AbsorbPlan absorb_plan(long long BH, int n_tokens, int sms) {
  const int tiles = ceil_div(n_tokens, hf::kAbsTok);
  int nsplit = BH >= sms ? 1 : static_cast<int>(sms / BH);
  if (nsplit > tiles) nsplit = tiles;
  if (nsplit < 1) nsplit = 1;
  const int per = ceil_div(tiles, nsplit);
  return AbsorbPlan{per, ceil_div(tiles, per)};
}

size_t absorb_ws_bytes(int B, int H, int n_tokens, int d) {
  const long long bh = static_cast<long long>(B) * H;
  const AbsorbPlan pl = absorb_plan(bh, n_tokens, kAbsorbTargetCtas);
  return align256(static_cast<size_t>(bh) * pl.nsplit * d * d * 4) +
         align256(static_cast<size_t>(bh) * pl.nsplit * d * 4);
}

// wait_first: 1 when the absorbed tokens may come from the previous kernel of the stream;
// 0 when the caller has ordered them before the previous kernel's start (the partial sums
// may then run beside that kernel's last CTAs, and only the slice reduction, which writes
// S and z, waits for it).
template <int D>
hf_status launch_absorb(hf_state* st, const hf_bf16* K_ev, const hf_bf16* V_ev, int n_tokens, void* ws,
                        cudaStream_t stream, int wait_first) {
  using C = hf::AbsorbCfg<D>;
  const long long BH = static_cast<long long>(st->B) * st->H;
  const AbsorbPlan pl = absorb_plan(BH, n_tokens, kAbsorbTargetCtas);
  CUtensorMap mk, mv;
  if (make_map(&mk, K_ev, D, n_tokens, BH, hf::kAbsTok) != HF_OK) return HF_ERR_CUDA;
  if (make_map(&mv, V_ev, D, n_tokens, BH, hf::kAbsTok) != HF_OK) return HF_ERR_CUDA;
  hf::AbsorbParams p;
  p.part_S = static_cast<float*>(ws);
  p.part_z = reinterpret_cast<float*>(static_cast<char*>(ws) +
                                      align256(static_cast<size_t>(BH) * pl.nsplit * D * D * 4));
  p.n_tokens = n_tokens;
  p.tiles_per_split = pl.tiles_per_split;
  p.nsplit = pl.nsplit;
  p.wait_first = wait_first;
  take_injection(2, &p.inject, &p.timeout_ns);
  if (cudaFuncSetAttribute(hf::absorb_partial_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           C::kDynSmem) != cudaSuccess)
    return HF_ERR_CUDA;
  if (launch_pdl(hf::absorb_partial_kernel<D>, BH * pl.nsplit, hf::kAbsThreads, C::kDynSmem, stream, mk, mv, p) !=
      HF_OK)
    return HF_ERR_CUDA;
  constexpr int kCtasPerHead = (D * D / 4 + 255) / 256;
  return launch_pdl(hf::reduce_state_kernel<D>, BH * kCtasPerHead, 256, 0, stream, st->S, st->z,
                    static_cast<uint8_t*>(st->S_split), static_cast<const float*>(p.part_S),
                    static_cast<const float*>(p.part_z), pl.nsplit);
}

// ---------------------------------------------------------------- attention
template <int D, int BLK, bool kRope = false>
hf_status launch_attn(const hf_bf16* Q, const hf_bf16* K, const hf_bf16* V, int BH, int Nq, int Nk, int r,
                      const int32_t* idx, const hf_state* st, float scale, hf_bf16* O, cudaStream_t stream,
                      const hf_rope* rope = nullptr) {
  using C = hf::AttnCfg<D, BLK, kRope>;
  const int nQB = ceil_div(Nq, BLK), nKB = ceil_div(Nk, BLK);
  CUtensorMap mq, mk, mv, mo;
  if (make_map(&mq, Q, D, Nq, BH, 128) != HF_OK || make_map(&mk, K, D, Nk, BH, BLK) != HF_OK ||
      make_map(&mv, V, D, Nk, BH, BLK) != HF_OK || make_map(&mo, O, D, Nq, BH, BLK) != HF_OK)
    return HF_ERR_CUDA;
  hf::AttnParams p;
  p.idx = idx;
  p.S_split = static_cast<const uint8_t*>(st->S_split);
  p.z = st->z;
  p.nQB = nQB;
  p.nKB = nKB;
  p.r = r;
  p.last_len = Nk - (nKB - 1) * BLK;
  p.scale_log2 = scale * 1.4426950408889634f;
  take_injection(3, &p.inject, &p.timeout_ns);
  p.rope_dt = p.rope_T = p.q_frame0 = p.n_frames = p.rope_cap = 0;
  p.rope_log2base = 0.f;
  if (kRope) {
    p.rope_dt = rope->d_t;
    p.rope_T = rope->tokens_per_frame;
    p.q_frame0 = rope->q_frame0;
    p.n_frames = ceil_div(Nk, rope->tokens_per_frame);
    p.rope_cap = rope->cap;
    p.rope_log2base = std::log2(rope->base);
  }
  if (cudaFuncSetAttribute(hf::hybrid_attn_kernel<D, BLK, kRope>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           C::kDynSmem) != cudaSuccess)
    return HF_ERR_CUDA;
  return launch_pdl(hf::hybrid_attn_kernel<D, BLK, kRope>, static_cast<long long>(BH) * nQB,
                    kRope ? hf::kAttnThreadsRope : hf::kAttnThreads, C::kDynSmem, stream, mq, mk, mv, mo, p);
}

}  // namespace

// ---------------------------------------------------------------- select without a caller workspace
// Scratch of hf_select_blocks_noalloc: the pooled Q and K rows of one call, in place of
// the caller's workspace. One copy per device (a module-scope __device__ array), so the
// call needs no allocation; its address on a device is looked up once, with that device
// current, and cached.
static __device__ __align__(256) unsigned char g_select_scratch[HF_SELECT_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kScratchMaxDevices = 64;
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
std::mutex g_scratch_mu;
// Per device: the context the address was looked up in, and the address. A symbol has
// one copy per context, so a lookup made in another context (a non-primary context, or a
// primary context created anew after cudaDeviceReset) is not reused.
struct ScratchEntry {
  CUcontext ctx = nullptr;
  void* ptr = nullptr;
};
ScratchEntry g_scratch[kScratchMaxDevices];

// Device address of g_select_scratch in the current context (set-up on first use there).
hf_status select_scratch(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return HF_ERR_CUDA;
  if (dev < 0 || dev >= kScratchMaxDevices) return HF_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  static CtxGetCurrentFn ctx_get = nullptr;
  if (!ctx_get) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
      return HF_ERR_CUDA;
    ctx_get = reinterpret_cast<CtxGetCurrentFn>(fn);
  }
  // cudaGetDevice above made the device's primary context current when none was
  CUcontext ctx = nullptr;
  if (ctx_get(&ctx) != CUDA_SUCCESS || !ctx) return HF_ERR_CUDA;
  ScratchEntry& e = g_scratch[dev];
  if (!e.ptr || e.ctx != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_select_scratch) != cudaSuccess || !p) return HF_ERR_CUDA;
    e.ctx = ctx;
    e.ptr = p;
  }
  *out = e.ptr;
  return HF_OK;
}

}  // namespace

namespace {

// Argument checks of hf_hybrid_attn_fwd (nothing is launched).
hf_status check_attn_args(const hf_bf16* Q, const hf_bf16* K, const hf_bf16* V, int B, int H, int Nq, int Nk, int d,
                          int block, int r, const int32_t* idx, const hf_state* st, float scale, const hf_bf16* O) {
  if (B < 1 || H < 1 || Nq < 0 || Nk < 1 || !st) return HF_ERR_INVALID_ARG;
  if (!supported_d(d) || !supported_block(block)) return HF_ERR_UNSUPPORTED;
  const int nKB = ceil_div(Nk, block);
  if (r < 1 || r > nKB) return HF_ERR_INVALID_ARG;
  if (st->B != B || st->H != H || st->d != d || !st->S || !st->z || !st->S_split) return HF_ERR_INVALID_ARG;
  if (!(scale == scale) || std::isinf(scale)) return HF_ERR_INVALID_ARG;
  if (Nq == 0) return HF_OK;
  if (!Q || !K || !V || !idx || !O) return HF_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(idx) || !aligned16(st->S) ||
      !aligned16(st->z) || !aligned16(st->S_split))
    return HF_ERR_ALIGNMENT;
  if (static_cast<long long>(B) * H * ceil_div(Nq, block) > 0x7fffffffLL) return HF_ERR_UNSUPPORTED;
  return HF_OK;
}

// Argument checks of hf_absorb_evicted for n_tokens >= 1 (nothing is launched).
hf_status check_absorb_args(const hf_state* st, const hf_bf16* K_ev, const hf_bf16* V_ev, int n_tokens,
                            const void* ws, size_t ws_bytes) {
  if (!st || !st->S || !st->z || !st->S_split || st->B < 1 || st->H < 1 || n_tokens < 0) return HF_ERR_INVALID_ARG;
  if (!supported_d(st->d)) return HF_ERR_UNSUPPORTED;
  if (n_tokens == 0) return HF_OK;
  if (!K_ev || !V_ev) return HF_ERR_INVALID_ARG;
  if (!aligned16(K_ev) || !aligned16(V_ev) || !aligned16(st->S) || !aligned16(st->z) || !aligned16(st->S_split))
    return HF_ERR_ALIGNMENT;
  const size_t need = absorb_ws_bytes(st->B, st->H, n_tokens, st->d);
  if (!ws || ws_bytes < need) return HF_ERR_WORKSPACE;
  if (!aligned16(ws)) return HF_ERR_ALIGNMENT;
  return HF_OK;
}

// The attention launch for already-checked arguments with Nq >= 1 (rope: the temporal
// RoPE variant, or NULL).
hf_status dispatch_attn(const hf_bf16* Q, const hf_bf16* K, const hf_bf16* V, int B, int H, int Nq, int Nk, int d,
                        int block, int r, const int32_t* idx, const hf_state* st, float scale, hf_bf16* O,
                        cudaStream_t s, const hf_rope* rope = nullptr) {
  const float sc = scale > 0.f ? scale : 1.0f / std::sqrt(static_cast<float>(d));
  const int bh = B * H;
#define HF_ATTN_CASE(DD, BB)                                                                               \
  if (d == DD && block == BB)                                                                              \
    return rope ? launch_attn<DD, BB, true>(Q, K, V, bh, Nq, Nk, r, idx, st, sc, O, s, rope)                \
                : launch_attn<DD, BB>(Q, K, V, bh, Nq, Nk, r, idx, st, sc, O, s);
  HF_ATTN_CASE(128, 128)
  HF_ATTN_CASE(128, 64)
  HF_ATTN_CASE(128, 32)
  HF_ATTN_CASE(64, 128)
  HF_ATTN_CASE(64, 64)
  HF_ATTN_CASE(64, 32)
#undef HF_ATTN_CASE
  return HF_ERR_UNSUPPORTED;
}

}  // namespace

extern "C" {

HF_API const char* hf_version(void) { return "hf-b200 0.1.0 (sm_100a)"; }

HF_API const char* hf_status_string(hf_status s) {
  switch (s) {
    case HF_OK: return "HF_OK";
    case HF_ERR_INVALID_ARG: return "HF_ERR_INVALID_ARG: invalid argument";
    case HF_ERR_UNSUPPORTED: return "HF_ERR_UNSUPPORTED: d must be 64 or 128, block 32, 64 or 128";
    case HF_ERR_ALIGNMENT: return "HF_ERR_ALIGNMENT: pointers must be 16-byte aligned";
    case HF_ERR_WORKSPACE: return "HF_ERR_WORKSPACE: workspace missing or too small";
    case HF_ERR_CUDA: return "HF_ERR_CUDA: a CUDA call or kernel launch failed";
    case HF_ERR_DEVICE_TIMEOUT: return "HF_ERR_DEVICE_TIMEOUT: a kernel gave up on an internal wait";
    case HF_ERR_DEVICE_BAD_INDEX: return "HF_ERR_DEVICE_BAD_INDEX: a block index outside [0, nKB) was skipped";
  }
  return "unknown hf_status";
}

HF_API size_t hf_workspace_size(int which, int B, int H, int Nq, int Nk, int d, int block, int r) {
  if (B < 1 || H < 1 || !supported_d(d)) return static_cast<size_t>(-1);
  switch (which) {
    case HF_WS_SELECT:
      if (!supported_block(block) || Nq < 0 || Nk < 1 || r < 1 || r > ceil_div(Nk, block))
        return static_cast<size_t>(-1);
      return select_ws_bytes(B, H, Nq, Nk, d, block);
    case HF_WS_ATTN:
      if (!supported_block(block) || Nq < 0 || Nk < 1 || r < 1 || r > ceil_div(Nk, block))
        return static_cast<size_t>(-1);
      return 0;
    case HF_WS_ABSORB:
      if (Nk < 0) return static_cast<size_t>(-1);
      if (Nk == 0) return 0;
      return absorb_ws_bytes(B, H, Nk, d);
    case HF_WS_SELECT_TWO_STAGE:
      if (!supported_block(block) || Nq < 0 || Nk < 1 || r < 1 || r > ceil_div(Nk, block))
        return static_cast<size_t>(-1);
      return select2_ws_bytes(B, H, Nq, Nk, d, block);
  }
  return static_cast<size_t>(-1);
}

HF_API hf_status hf_state_init(hf_state* st, int B, int H, int d, float* S_dev, float* z_dev, void* S_split_dev,
                               void* stream) {
  if (!st || !S_dev || !z_dev || !S_split_dev || B < 1 || H < 1) return HF_ERR_INVALID_ARG;
  if (!supported_d(d)) return HF_ERR_UNSUPPORTED;
  if (!aligned16(S_dev) || !aligned16(z_dev) || !aligned16(S_split_dev)) return HF_ERR_ALIGNMENT;
  const size_t bh = static_cast<size_t>(B) * H;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(S_dev, 0, bh * d * d * sizeof(float), s) != cudaSuccess) return HF_ERR_CUDA;
  if (cudaMemsetAsync(z_dev, 0, bh * d * sizeof(float), s) != cudaSuccess) return HF_ERR_CUDA;
  if (cudaMemsetAsync(S_split_dev, 0, HF_STATE_SPLIT_BYTES(B, H, d), s) != cudaSuccess) return HF_ERR_CUDA;
  st->B = B;
  st->H = H;
  st->d = d;
  st->S = S_dev;
  st->z = z_dev;
  st->S_split = S_split_dev;
  st->n_absorbed = 0;
  return HF_OK;
}

HF_API hf_status hf_absorb_evicted(hf_state* st, const hf_bf16* K_ev, const hf_bf16* V_ev, int n_tokens, void* ws,
                                   size_t ws_bytes, void* stream) {
  const hf_status chk = check_absorb_args(st, K_ev, V_ev, n_tokens, ws, ws_bytes);
  if (chk != HF_OK || n_tokens == 0) return chk;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const hf_status rc = st->d == 128 ? launch_absorb<128>(st, K_ev, V_ev, n_tokens, ws, s, 1)
                                    : launch_absorb<64>(st, K_ev, V_ev, n_tokens, ws, s, 1);
  if (rc == HF_OK) st->n_absorbed += n_tokens;
  return rc;
}

HF_API hf_status hf_select_blocks(const hf_bf16* Q, const hf_bf16* K, int B, int H, int Nq, int Nk, int d,
                                  int block, int r, int32_t* idx_out, float* scores_out, void* ws,
                                  size_t ws_bytes, void* stream) {
  if (B < 1 || H < 1 || Nq < 0 || Nk < 1) return HF_ERR_INVALID_ARG;
  if (!supported_d(d) || !supported_block(block)) return HF_ERR_UNSUPPORTED;
  const int nKB = ceil_div(Nk, block);
  if (r < 1 || r > nKB) return HF_ERR_INVALID_ARG;
  if (nKB > hf::kMaxKeyBlocks) return HF_ERR_UNSUPPORTED;
  if (Nq == 0) return HF_OK;
  if (!Q || !K || !idx_out) return HF_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(idx_out) || (scores_out && !aligned16(scores_out)))
    return HF_ERR_ALIGNMENT;
  if (!ws || ws_bytes < select_ws_bytes(B, H, Nq, Nk, d, block)) return HF_ERR_WORKSPACE;
  if (!aligned16(ws)) return HF_ERR_ALIGNMENT;
  const long long BH = static_cast<long long>(B) * H;
  if (!select_grid_ok(BH, Nq, nKB, block)) return HF_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return d == 128 ? launch_select<128>(Q, K, static_cast<int>(BH), Nq, Nk, block, r, idx_out, scores_out, ws, s)
                  : launch_select<64>(Q, K, static_cast<int>(BH), Nq, Nk, block, r, idx_out, scores_out, ws, s);
}

HF_API hf_status hf_select_blocks_rope(const hf_bf16* Q, const hf_bf16* K, int B, int H, int Nq, int Nk, int d,
                                       int block, int r, const hf_rope* rope, int32_t* idx_out, float* scores_out,
                                       void* ws, size_t ws_bytes, void* stream) {
  if (B < 1 || H < 1 || Nq < 0 || Nk < 1) return HF_ERR_INVALID_ARG;
  if (!supported_d(d) || !supported_block(block)) return HF_ERR_UNSUPPORTED;
  const int nKB = ceil_div(Nk, block);
  if (r < 1 || r > nKB) return HF_ERR_INVALID_ARG;
  if (nKB > hf::kMaxKeyBlocks) return HF_ERR_UNSUPPORTED;
  if (!rope_ok(rope, d, Nq, Nk, block)) return HF_ERR_INVALID_ARG;
  if (Nq == 0) return HF_OK;
  if (!Q || !K || !idx_out) return HF_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(idx_out) || (scores_out && !aligned16(scores_out)))
    return HF_ERR_ALIGNMENT;
  if (!ws || ws_bytes < select_ws_bytes(B, H, Nq, Nk, d, block)) return HF_ERR_WORKSPACE;
  if (!aligned16(ws)) return HF_ERR_ALIGNMENT;
  const long long BH = static_cast<long long>(B) * H;
  if (!select_grid_ok(BH, Nq, nKB, block)) return HF_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return d == 128
             ? launch_select<128>(Q, K, static_cast<int>(BH), Nq, Nk, block, r, idx_out, scores_out, ws, s, rope)
             : launch_select<64>(Q, K, static_cast<int>(BH), Nq, Nk, block, r, idx_out, scores_out, ws, s, rope);
}

// ---------------------------------------------------------------- pooled-key cache
HF_API hf_status hf_kpool_init(hf_kpool* kp, int B, int H, int d, int granule, int capacity, float* sums_dev) {
  if (!kp || B < 1 || H < 1 || capacity < 1 || capacity > (1 << 30) || !sums_dev) return HF_ERR_INVALID_ARG;
  if (granule < 1 || granule > 128 || (128 % granule) != 0) return HF_ERR_INVALID_ARG;
  if (!supported_d(d)) return HF_ERR_UNSUPPORTED;
  if (!aligned16(sums_dev)) return HF_ERR_ALIGNMENT;
  if (static_cast<long long>(B) * H > 0x7fffffffLL) return HF_ERR_UNSUPPORTED;
  kp->B = B;
  kp->H = H;
  kp->d = d;
  kp->granule = granule;
  kp->capacity = capacity;
  kp->n_gran = 0;
  kp->head = 0;
  kp->sums = sums_dev;
  return HF_OK;
}

// The window after a push (validated; kp unchanged) and the push's kernel arguments.
struct PushPlan {
  int head, n_gran;     // the window after the push
  hf::PushArgs args;    // n_new == 0: no device work
  long long ctas;       // push CTAs
};

static hf_status plan_push(const hf_kpool* kp, const hf_bf16* K_new, int n_tokens, int n_evict, PushPlan* pl) {
  if (!kp || !kp->sums || kp->B < 1 || kp->H < 1 || kp->capacity < 1 || kp->granule < 1) return HF_ERR_INVALID_ARG;
  if (!supported_d(kp->d)) return HF_ERR_UNSUPPORTED;
  const int G = kp->granule, cap = kp->capacity;
  if (n_tokens < 0 || n_evict < 0 || n_tokens % G != 0 || n_evict % G != 0) return HF_ERR_INVALID_ARG;
  if (kp->n_gran < 0 || kp->n_gran > cap || kp->head < 0 || kp->head >= cap) return HF_ERR_INVALID_ARG;
  const int ev = n_evict / G, n_new = n_tokens / G;
  if (ev > kp->n_gran || kp->n_gran - ev + n_new > cap) return HF_ERR_INVALID_ARG;
  if (n_new > 0 && !K_new) return HF_ERR_INVALID_ARG;
  if (n_new > 0 && !aligned16(K_new)) return HF_ERR_ALIGNMENT;
  const int head = (kp->head + ev) % cap, kept = kp->n_gran - ev;
  constexpr int kGran128 = hf::kPoolThreads / (128 / 8), kGran64 = hf::kPoolThreads / (64 / 8);
  const int per_cta = kp->d == 128 ? kGran128 : kGran64;
  const long long BH = static_cast<long long>(kp->B) * kp->H;
  pl->ctas = n_new > 0 ? BH * ((n_new + per_cta - 1) / per_cta) : 0;
  if (pl->ctas > 0x7fffffffLL) return HF_ERR_UNSUPPORTED;
  pl->head = head;
  pl->n_gran = kept + n_new;
  pl->args = hf::PushArgs{reinterpret_cast<const __nv_bfloat16*>(K_new), n_tokens, G, n_new, (head + kept) % cap,
                          cap, kp->sums};
  return HF_OK;
}

HF_API hf_status hf_kpool_push(hf_kpool* kp, const hf_bf16* K_new, int n_tokens, int n_evict, void* stream) {
  PushPlan pl;
  const hf_status rc = plan_push(kp, K_new, n_tokens, n_evict, &pl);
  if (rc != HF_OK) return rc;
  if (pl.ctas > 0) {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const hf_status lr = kp->d == 128 ? launch_pdl(hf::kpool_push_kernel<128>, pl.ctas, hf::kPoolThreads, 0, s, pl.args)
                                      : launch_pdl(hf::kpool_push_kernel<64>, pl.ctas, hf::kPoolThreads, 0, s, pl.args);
    if (lr != HF_OK) return HF_ERR_CUDA;
  }
  kp->head = pl.head;
  kp->n_gran = pl.n_gran;
  return HF_OK;
}

// Checks of a cached selection over the window of kp; *Nk_out: its key tokens.
static hf_status check_select_cached(const hf_bf16* Q, const hf_kpool* kp, int Nq, int block, int r,
                                     const int32_t* idx_out, const float* scores_out, const void* ws,
                                     size_t ws_bytes, int* Nk_out) {
  if (!kp || !kp->sums || kp->B < 1 || kp->H < 1 || kp->granule < 1 || Nq < 0) return HF_ERR_INVALID_ARG;
  if (kp->n_gran < 1 || kp->n_gran > kp->capacity || kp->head < 0 || kp->head >= kp->capacity)
    return HF_ERR_INVALID_ARG;
  if (!supported_d(kp->d) || !supported_block(block)) return HF_ERR_UNSUPPORTED;
  if (block % kp->granule != 0) return HF_ERR_INVALID_ARG;
  const long long nk = static_cast<long long>(kp->n_gran) * kp->granule;
  if (nk > 0x7fffffffLL) return HF_ERR_UNSUPPORTED;
  const int Nk = static_cast<int>(nk), B = kp->B, H = kp->H, d = kp->d;
  const int nKB = ceil_div(Nk, block);
  if (r < 1 || r > nKB) return HF_ERR_INVALID_ARG;
  if (nKB > hf::kMaxKeyBlocks) return HF_ERR_UNSUPPORTED;
  *Nk_out = Nk;
  if (Nq == 0) return HF_OK;
  if (!Q || !idx_out) return HF_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(idx_out) || (scores_out && !aligned16(scores_out))) return HF_ERR_ALIGNMENT;
  if (!ws || ws_bytes < select_ws_bytes(B, H, Nq, Nk, d, block)) return HF_ERR_WORKSPACE;
  if (!aligned16(ws)) return HF_ERR_ALIGNMENT;
  const long long BH = static_cast<long long>(B) * H;
  if (BH * (ceil_div(Nq, block) + nKB) > 0x7fffffffLL) return HF_ERR_UNSUPPORTED;
  return HF_OK;
}

HF_API hf_status hf_select_blocks_cached(const hf_bf16* Q, const hf_kpool* kp, int Nq, int block, int r,
                                         int32_t* idx_out, float* scores_out, void* ws, size_t ws_bytes,
                                         void* stream) {
  int Nk = 0;
  const hf_status rc = check_select_cached(Q, kp, Nq, block, r, idx_out, scores_out, ws, ws_bytes, &Nk);
  if (rc != HF_OK || Nq == 0) return rc;
  const int BH = kp->B * kp->H;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return kp->d == 128 ? launch_select_cached<128>(Q, kp, BH, Nq, Nk, block, r, idx_out, scores_out, ws, s)
                      : launch_select_cached<64>(Q, kp, BH, Nq, Nk, block, r, idx_out, scores_out, ws, s);
}

HF_API hf_status hf_select_blocks_cached_push(const hf_bf16* Q, hf_kpool* kp, const hf_bf16* K_new, int n_tokens,
                                              int n_evict, int Nq, int block, int r, int32_t* idx_out,
                                              float* scores_out, void* ws, size_t ws_bytes, void* stream) {
  PushPlan pl;
  hf_status rc = plan_push(kp, K_new, n_tokens, n_evict, &pl);
  if (rc != HF_OK) return rc;
  hf_kpool after = *kp;
  after.head = pl.head;
  after.n_gran = pl.n_gran;
  int Nk = 0;
  rc = check_select_cached(Q, &after, Nq, block, r, idx_out, scores_out, ws, ws_bytes, &Nk);
  if (rc != HF_OK) return rc;
  const int BH = kp->B * kp->H;
  if (static_cast<long long>(BH) * ceil_div(Nq, block) + pl.ctas > 0x7fffffffLL) return HF_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (Nq == 0) {
    // nothing to select: the push alone
    return hf_kpool_push(kp, K_new, n_tokens, n_evict, stream);
  }
  const hf::PushArgs* push = pl.ctas > 0 ? &pl.args : nullptr;
  rc = kp->d == 128
           ? launch_select_cached<128>(Q, &after, BH, Nq, Nk, block, r, idx_out, scores_out, ws, s, push, pl.ctas)
           : launch_select_cached<64>(Q, &after, BH, Nq, Nk, block, r, idx_out, scores_out, ws, s, push, pl.ctas);
  if (rc != HF_OK) return rc;
  *kp = after;
  return HF_OK;
}

HF_API hf_status hf_select_blocks_two_stage(const hf_bf16* Q, const hf_bf16* K, int B, int H, int Nq, int Nk,
                                            int d, int block, int r, int tokens_per_frame, int n_frames,
                                            int32_t* idx_out, int32_t* frames_out, float* scores_out, void* ws,
                                            size_t ws_bytes, void* stream) {
  if (B < 1 || H < 1 || Nq < 0 || Nk < 1) return HF_ERR_INVALID_ARG;
  if (!supported_d(d) || !supported_block(block)) return HF_ERR_UNSUPPORTED;
  if (tokens_per_frame < block) return HF_ERR_INVALID_ARG;
  const int nKB = ceil_div(Nk, block), W = ceil_div(Nk, tokens_per_frame);
  if (r < 1 || r > nKB || n_frames < 1 || n_frames > W) return HF_ERR_INVALID_ARG;
  if (nKB > hf::kMaxKeyBlocks2) return HF_ERR_UNSUPPORTED;
  if (Nq == 0) return HF_OK;
  if (!Q || !K || !idx_out) return HF_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(idx_out) || (frames_out && !aligned16(frames_out)) ||
      (scores_out && !aligned16(scores_out)))
    return HF_ERR_ALIGNMENT;
  if (!ws || ws_bytes < select2_ws_bytes(B, H, Nq, Nk, d, block)) return HF_ERR_WORKSPACE;
  if (!aligned16(ws)) return HF_ERR_ALIGNMENT;
  const long long BH = static_cast<long long>(B) * H;
  if (BH * (ceil_div(Nq, block) + nKB) > 0x7fffffffLL) return HF_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return d == 128 ? launch_select2<128>(Q, K, static_cast<int>(BH), Nq, Nk, block, r, tokens_per_frame, n_frames,
                                        idx_out, frames_out, scores_out, ws, s)
                  : launch_select2<64>(Q, K, static_cast<int>(BH), Nq, Nk, block, r, tokens_per_frame, n_frames,
                                       idx_out, frames_out, scores_out, ws, s);
}

HF_API hf_status hf_hybrid_attn_fwd(const hf_bf16* Q, const hf_bf16* K, const hf_bf16* V, int B, int H, int Nq,
                                    int Nk, int d, int block, int r, const int32_t* idx, const hf_state* st,
                                    float scale, hf_bf16* O, void* ws, size_t ws_bytes, void* stream) {
  (void)ws;
  (void)ws_bytes;
  const hf_status rc = check_attn_args(Q, K, V, B, H, Nq, Nk, d, block, r, idx, st, scale, O);
  if (rc != HF_OK || Nq == 0) return rc;
  return dispatch_attn(Q, K, V, B, H, Nq, Nk, d, block, r, idx, st, scale, O, static_cast<cudaStream_t>(stream));
}

HF_API hf_status hf_hybrid_attn_fwd_rope(const hf_bf16* Q, const hf_bf16* K, const hf_bf16* V, int B, int H,
                                         int Nq, int Nk, int d, int block, int r, const int32_t* idx,
                                         const hf_state* st, float scale, const hf_rope* rope, hf_bf16* O, void* ws,
                                         size_t ws_bytes, void* stream) {
  (void)ws;
  (void)ws_bytes;
  const hf_status rc = check_attn_args(Q, K, V, B, H, Nq, Nk, d, block, r, idx, st, scale, O);
  if (rc != HF_OK) return rc;
  if (!rope_ok(rope, d, Nq, Nk, block)) return HF_ERR_INVALID_ARG;
  if (Nq == 0) return HF_OK;
  return dispatch_attn(Q, K, V, B, H, Nq, Nk, d, block, r, idx, st, scale, O, static_cast<cudaStream_t>(stream),
                       rope);
}

HF_API hf_status hf_hybrid_attn_fwd_absorb(const hf_bf16* Q, const hf_bf16* K, const hf_bf16* V, int B, int H,
                                           int Nq, int Nk, int d, int block, int r, const int32_t* idx, hf_state* st,
                                           float scale, hf_bf16* O, const hf_bf16* K_ev, const hf_bf16* V_ev,
                                           int n_evicted, void* ws, size_t ws_bytes, void* stream) {
  hf_status rc = check_attn_args(Q, K, V, B, H, Nq, Nk, d, block, r, idx, st, scale, O);
  if (rc != HF_OK) return rc;
  rc = check_absorb_args(st, K_ev, V_ev, n_evicted, ws, ws_bytes);
  if (rc != HF_OK) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int wait_first = 1;  // without an attention launch before it, the absorption waits as on its own
  if (Nq > 0) {
    rc = dispatch_attn(Q, K, V, B, H, Nq, Nk, d, block, r, idx, st, scale, O, s);
    if (rc != HF_OK) return rc;
    wait_first = 0;
  }
  if (n_evicted == 0) return HF_OK;
  rc = d == 128 ? launch_absorb<128>(st, K_ev, V_ev, n_evicted, ws, s, wait_first)
                : launch_absorb<64>(st, K_ev, V_ev, n_evicted, ws, s, wait_first);
  if (rc == HF_OK) st->n_absorbed += n_evicted;
  return rc;
}

HF_API hf_status hf_keep_schedule(int n_chunks, const int* nKB, double s_base, double s_target, int* r_out,
                                  double* s_out, double* beta_out) {
  if (n_chunks < 1 || !nKB || !r_out) return HF_ERR_INVALID_ARG;
  if (!(s_base >= 0.0 && s_base < 1.0) || !(s_target >= 0.0 && s_target < 1.0)) return HF_ERR_INVALID_ARG;
  double total = 0.0, later = 0.0, later_w = 0.0;  // all blocks; chunks >= 1; weighted by 1/sqrt(i)
  for (int i = 0; i < n_chunks; ++i) {
    if (nKB[i] < 1) return HF_ERR_INVALID_ARG;
    total += nKB[i];
    if (i > 0) {
      later += nKB[i];
      later_w += nKB[i] / std::sqrt(static_cast<double>(i));
    }
  }
  // (1 - s_target) total = nKB[0] + (1 - s_base) later + beta later_w
  const double beta = n_chunks > 1 ? ((1.0 - s_target) * total - nKB[0] - (1.0 - s_base) * later) / later_w : 0.0;
  if (!(beta >= 0.0)) return HF_ERR_INVALID_ARG;
  std::vector<double> s(n_chunks, 0.0);
  for (int i = 1; i < n_chunks; ++i) {
    s[i] = s_base - beta / std::sqrt(static_cast<double>(i));
    if (!(s[i] >= 0.0 && s[i] < 1.0)) return HF_ERR_INVALID_ARG;
  }
  for (int i = 0; i < n_chunks; ++i) {
    const double keep = std::ceil((1.0 - s[i]) * nKB[i]);
    r_out[i] = keep < 1.0 ? 1 : (keep > nKB[i] ? nKB[i] : static_cast<int>(keep));
    if (s_out) s_out[i] = s[i];
  }
  if (beta_out) *beta_out = beta;
  return HF_OK;
}

HF_API hf_status hf_query_status(void* stream, uint32_t* detail_out) {
  if (detail_out) *detail_out = 0;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return HF_ERR_CUDA;
  uint32_t word = 0;
  if (cudaMemcpyFromSymbol(&word, hf::g_hf_error_word, sizeof(word)) != cudaSuccess) return HF_ERR_CUDA;
  if (word == 0) return HF_OK;
  const uint32_t zero = 0;
  if (cudaMemcpyToSymbol(hf::g_hf_error_word, &zero, sizeof(zero)) != cudaSuccess) return HF_ERR_CUDA;
  if (detail_out) *detail_out = word;
  return (word >> 16) == 0x7200u ? HF_ERR_DEVICE_BAD_INDEX : HF_ERR_DEVICE_TIMEOUT;
}

HF_API hf_status hf_debug_inject_timeout(int kernel_id, int count, unsigned long long timeout_ns) {
  if (kernel_id < 0 || kernel_id > 3 || count < 0) return HF_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_mu);
  g_inject.kernel_id = (kernel_id == 0 || count == 0) ? 0 : kernel_id;
  g_inject.count = count;
  g_inject.timeout_ns = timeout_ns ? timeout_ns : kDefaultTimeoutNs;
  return HF_OK;
}

HF_API hf_status hf_select_blocks_noalloc(const hf_bf16* Q, const hf_bf16* K, int B, int H, int Nq, int Nk,
                                          int d, int block, int r, int32_t* idx_out, float* scores_out,
                                          void* stream) {
  // Every argument check of hf_select_blocks, then the size check against the fixed
  // scratch, all before the set-up: a rejected call makes no CUDA call at all.
  if (B < 1 || H < 1 || Nq < 0 || Nk < 1) return HF_ERR_INVALID_ARG;
  if (!supported_d(d) || !supported_block(block)) return HF_ERR_UNSUPPORTED;
  const int nKB = ceil_div(Nk, block);
  if (r < 1 || r > nKB) return HF_ERR_INVALID_ARG;
  if (nKB > hf::kMaxKeyBlocks) return HF_ERR_UNSUPPORTED;
  if (Nq == 0) return HF_OK;
  if (!Q || !K || !idx_out) return HF_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(idx_out) || (scores_out && !aligned16(scores_out)))
    return HF_ERR_ALIGNMENT;
  if (!select_grid_ok(static_cast<long long>(B) * H, Nq, nKB, block)) return HF_ERR_UNSUPPORTED;
  const size_t need = select_ws_bytes(B, H, Nq, Nk, d, block);
  if (need > HF_SELECT_NOALLOC_SCRATCH_BYTES) return HF_ERR_WORKSPACE;
  void* scratch = nullptr;
  const hf_status rc = select_scratch(&scratch);
  if (rc != HF_OK) return rc;
  return hf_select_blocks(Q, K, B, H, Nq, Nk, d, block, r, idx_out, scores_out, scratch,
                          HF_SELECT_NOALLOC_SCRATCH_BYTES, stream);
}

HF_API unsigned long long hf_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"

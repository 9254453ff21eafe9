// Block scoring and top-r selection (hf_select_blocks, hf_select_blocks_two_stage,
// hf_select_blocks_cached with hf_kpool_push).
//
// Source: "Light Forcing: Accelerating Autoregressive Video Diffusion via Sparse
// Attention", German technical summary, section 2.2 (query and key tokens are
// compressed by mean pooling at block level; key blocks are selected per query
// block); "Long-Horizon Streaming Video Generation via Hybrid Attention with
// Decoupled Distillation", German technical summary, section 2 A (only the most
// important, Top-K, blocks are computed). Light Forcing section 2.2 also gives the
// two-stage variant (frames by frame-pooled keys, then blocks within them).
//
// All on CUDA cores (the work is a streaming read of Q and K plus a tiny score matrix,
// so tensor cores would not help):
//   pool_blocks_kernel   one CTA per (b,h,block) of Q or K: fp32 mean of the valid rows.
//                        HBM-bound: reads Q and K once with 16-byte loads, 8 in flight
//                        per thread.
//   score_select_staged_kernel  the same with a head's pooled K means (written
//                        transposed by the pooling) staged in shared memory by bulk
//                        copies, when they fit (see there).
//   score_select_kernel  one CTA per (b,h, 4 query blocks): s_IJ = Qbar_I . Kbar_J, a
//                        thread per key block; then one warp per query block finds the
//                        r-th largest score by a bitwise search (per-lane counts, one warp
//                        reduction per bit), takes every block above it and the lowest-J
//                        blocks equal to it, and writes the r blocks in ascending J.
//                        NaN scores are ranked as -inf, so exactly r blocks are written.
// Two-stage selection: pool_blocks_kernel<d, true> also writes each key block's sums in
// its first and next frame, pool_frames_kernel adds them into frame means, and
// score_select2_kernel keeps frames first, then blocks within them (see there).
// Pooled-key cache: kpool_push_kernel sums each granule of G new keys into a ring, and
// kpool_blocks_kernel forms the window's key block means from those sums (see there).
// Every kernel is launched with programmatic stream serialisation: it waits for the
// previous grid of its stream before its first read and then lets the next one be
// scheduled (griddep_wait / griddep_launch_dependents in hf_ptx.cuh).
#pragma once

#include "hf_ptx.cuh"

namespace hf {

constexpr int kPoolThreads = 256;
constexpr int kSelectThreads = 256;
constexpr int kMaxKeyBlocks = 8192;  // 4 score rows of fp32 fit in shared memory

__device__ __forceinline__ void acc_bf16x8(float* acc, uint4 v) {
  acc[0] += bf16_lo_to_f32(v.x);
  acc[1] += bf16_hi_to_f32(v.x);
  acc[2] += bf16_lo_to_f32(v.y);
  acc[3] += bf16_hi_to_f32(v.y);
  acc[4] += bf16_lo_to_f32(v.z);
  acc[5] += bf16_hi_to_f32(v.z);
  acc[6] += bf16_lo_to_f32(v.w);
  acc[7] += bf16_hi_to_f32(v.w);
}

__device__ __forceinline__ uint4 ld_stream_16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

constexpr uint32_t kKernSelect = 1;

struct PoolArgs {
  const __nv_bfloat16* Q;
  const __nv_bfloat16* K;
  int Nq, Nk, block, nQB, nKB;
  float* Qp;     // [BH][nQB][D]
  float* Kp;     // [BH][nKB][D]
  int T;         // frame length in tokens (kParts, kRope)
  float* Kpart;  // [BH][nKB][2][D] (kParts)
  // temporal RoPE (kRope): Q's first token lies in window frame q_frame0, K's in frame 0;
  // the window holds n_frames frames; index cap; rotated dimensions [0, rope_dt); log2 of
  // the frequency base
  int q_frame0, n_frames, rope_cap, rope_dt;
  float rope_log2base;
  // 1: the key means go to Kp transposed, [BH][D][nKB] (for score_select_staged_kernel)
  int k_transposed;
};

// Temporal RoPE index of window frame w: the newest frame (n_frames - 1) at cap, every
// frame at least cap frames older at 0.
__device__ __forceinline__ int rope_index(int w, int n_frames, int cap) {
  return cap - min((n_frames - 1) - w, cap);
}

// (cos, sin) of the angle p * base^(-2i/d_t) of pair i (full-precision sincos).
__device__ __forceinline__ void rope_cs(int p, int i, int d_t, float log2base, float& c, float& s) {
  const float theta = exp2f(-static_cast<float>(2 * i) / static_cast<float>(d_t) * log2base);
  sincosf(static_cast<float>(p) * theta, &s, &c);
}

// Qp[bh][I][:] = mean of the Q rows of block I; Kp[bh][J][:] likewise for K. One CTA per
// (b, h, block): streaming 16-byte loads, 8 per thread in flight, then a reduction of the
// row phases through shared memory in a fixed order.
// kParts (two-stage selection): also Kpart[bh][J][0|1][:] = the sums of the rows of key
// block J that lie in its first frame (J*block / T) and in the next frame (zero when the
// block does not reach it); frames are runs of T >= block tokens, so a block touches at
// most two. The block means are computed exactly as without kParts.
// kRope: the rows of every block are summed per frame (a short second pass over the rows
// of the next frame, just read and still in L2), each frame's sum is turned by that
// frame's temporal RoPE index (pairs (2i, 2i+1) of the dimensions below d_t), and the mean
// is taken of the turned sums: the mean of the turned tokens, as the rotation is linear
// and one per frame.
template <int D>
struct PoolShape {
  static constexpr int kVec = 8;                     // bf16 per 16-byte load
  static constexpr int kTpr = D / kVec;              // threads per row
  static constexpr int kRows = kPoolThreads / kTpr;  // rows per pass
  static constexpr int kRedFloats = kRows * D;       // one row-phase reduction buffer
};

// The mean of block t of Q (is_key_block false) or K of head bh, computed by the whole
// CTA (kPoolThreads threads) with the reduction buffers red and red1 (kRedFloats each;
// red1 used with kParts or kRope), written by threads 0..D-1.
template <int D, bool kParts, bool kRope>
__device__ __forceinline__ void pool_block(const PoolArgs& a, int bh, int t, bool is_key_block, float* red,
                                           float* red1) {
  constexpr int kVec = PoolShape<D>::kVec;
  constexpr int kTpr = PoolShape<D>::kTpr;
  constexpr int kRows = PoolShape<D>::kRows;
  constexpr int kUnroll = 8;                    // loads in flight per thread
  constexpr bool kSplit = kParts || kRope;
  const __nv_bfloat16* X;
  int N;
  float* out;
  if (!is_key_block) {
    X = a.Q + static_cast<size_t>(bh) * a.Nq * D;
    N = a.Nq;
    out = a.Qp + (static_cast<size_t>(bh) * a.nQB + t) * D;
  } else {
    X = a.K + static_cast<size_t>(bh) * a.Nk * D;
    N = a.Nk;
    out = a.Kp + (static_cast<size_t>(bh) * a.nKB + t) * D;
  }
  const int lo = t * a.block;
  const int hi = min(lo + a.block, N);
  const int c = threadIdx.x % kTpr;
  const int rr = threadIdx.x / kTpr;
  // first row of the next frame, if this block reaches it (key blocks with kParts, every
  // block with kRope)
  const bool split = (kParts && is_key_block) || kRope;
  const int bnd = split ? min(hi, (lo / a.T + 1) * a.T) : hi;

  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int base = lo + rr; base < hi; base += kRows * kUnroll) {
    uint4 v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int row = base + u * kRows;
      v[u] = row < hi ? ld_stream_16(X + static_cast<size_t>(row) * D + c * kVec) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) acc_bf16x8(acc, v[u]);
  }
  // the second-frame sum, only in blocks that reach the next frame (CTA-uniform): a short
  // second pass over those rows, just read and still in L2
  float acc1[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if constexpr (kSplit) {
    if (bnd < hi) {
      for (int row = lo + rr; row < hi; row += kRows)
        if (row >= bnd) acc_bf16x8(acc1, ld_stream_16(X + static_cast<size_t>(row) * D + c * kVec));
    }
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) red[rr * D + c * kVec + k] = acc[k];
  if constexpr (kSplit) {
#pragma unroll
    for (int k = 0; k < 8; ++k) red1[rr * D + c * kVec + k] = acc1[k];
  }
  __syncthreads();
  float s = 0.f, s1 = 0.f;
  if (threadIdx.x < D) {
#pragma unroll 8
    for (int q = 0; q < kRows; ++q) s += red[q * D + threadIdx.x];
    if constexpr (kSplit) {
#pragma unroll 8
      for (int q = 0; q < kRows; ++q) s1 += red1[q * D + threadIdx.x];
    }
  }
  if constexpr (kRope) {
    // the two frames' sums, s - s1 and s1, turned by their indices; a pair (2i, 2i+1) needs
    // its partner column, exchanged through shared memory
    __syncthreads();
    if (threadIdx.x < D) {
      red[threadIdx.x] = s - s1;
      red[D + threadIdx.x] = s1;
    }
    __syncthreads();
    const int tc = threadIdx.x;
    if (tc < a.rope_dt) {
      const int i = tc >> 1;
      const int w0 = (is_key_block ? 0 : a.q_frame0) + lo / a.T;
      float r2[2];
#pragma unroll
      for (int f = 0; f < 2; ++f) {
        float cs, sn;
        rope_cs(rope_index(w0 + f, a.n_frames, a.rope_cap), i, a.rope_dt, a.rope_log2base, cs, sn);
        const float x0 = red[f * D + 2 * i], x1 = red[f * D + 2 * i + 1];
        r2[f] = (tc & 1) ? fmaf(x0, sn, x1 * cs) : fmaf(x0, cs, -x1 * sn);
      }
      s = r2[0] + r2[1];
      s1 = r2[1];
    }
  }
  if (threadIdx.x < D) {
    const float mean = s / static_cast<float>(hi - lo);
    if (is_key_block && a.k_transposed)
      a.Kp[(static_cast<size_t>(bh) * D + threadIdx.x) * a.nKB + t] = mean;
    else
      out[threadIdx.x] = mean;
    if constexpr (kParts) {
      if (is_key_block) {
        float* pt = a.Kpart + ((static_cast<size_t>(bh) * a.nKB + t) * 2) * D;
        pt[threadIdx.x] = s - s1;
        pt[D + threadIdx.x] = s1;
      }
    }
  }
}

// Eight CTAs per SM (2048 threads): the loads in flight fit in 32 registers a thread.
template <int D, bool kParts = false, bool kRope = false>
__global__ void __launch_bounds__(kPoolThreads, kRope ? 6 : 8) pool_blocks_kernel(PoolArgs a) {
  __shared__ float red[PoolShape<D>::kRedFloats];
  __shared__ float red1[(kParts || kRope) ? PoolShape<D>::kRedFloats : 1];
  griddep_wait();
  griddep_launch_dependents();
  const int per_bh = a.nQB + a.nKB;
  const int bh = blockIdx.x / per_bh;
  const int t = blockIdx.x % per_bh;
  if (t < a.nQB)
    pool_block<D, kParts, kRope>(a, bh, t, false, red, red1);
  else
    pool_block<D, kParts, kRope>(a, bh, t - a.nQB, true, red, red1);
}

// Kf[bh][w][:] = mean of the key rows of frame w (rows [w*T, min((w+1)*T, Nk))), summed
// from the block parts in block order (deterministic). One CTA per (bh, w), D threads.
template <int D>
__global__ void __launch_bounds__(D) pool_frames_kernel(const float* __restrict__ Kpart, int Nk, int block, int T,
                                                        int nKB, int W, float* __restrict__ Kf) {
  griddep_wait();
  griddep_launch_dependents();
  const int bh = blockIdx.x / W, w = blockIdx.x % W;
  const int f_lo = w * T, f_hi = min(f_lo + T, Nk);
  const int J_lo = f_lo / block, J_hi = (f_hi - 1) / block;
  const float* P = Kpart + static_cast<size_t>(bh) * nKB * 2 * D;
  float s = 0.f;
  for (int J = J_lo; J <= J_hi; ++J) {
    // block J starts in frame w (its first part) or in frame w-1 and reaches w (second)
    const int part = (J * block) / T == w ? 0 : 1;
    s += P[(static_cast<size_t>(J) * 2 + part) * D + threadIdx.x];
  }
  Kf[(static_cast<size_t>(bh) * W + w) * D + threadIdx.x] = s / static_cast<float>(f_hi - f_lo);
}

// Scores of kSelQB query blocks of one head per CTA (each pooled K row is read once for
// all of them), then one warp per query block selects its top r.
constexpr int kSelQB = 4;

// Order-preserving map of a float to an unsigned integer (NaN has been replaced by -inf).
__device__ __forceinline__ uint32_t ordered_bits(float f) {
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Warp-wide top-r over n unique keys key_at(J) (J < n): larger key first, lower J first on
// ties; emit(J, pos) is called for the r selected J in ascending J (pos = 0..r-1). Keys
// are order-preserving 32-bit codes; a key of 0 ranks below every real score code
// (ordered(-inf) = 0x007FFFFF), so it is chosen only when fewer than r keys are nonzero.
// NPL = keys per lane held in registers (lane l holds J = 32 k + l); NPL = 0 calls key_at
// each time (any n).
// 1. T = the r-th largest key: the largest t with #{J : key_J >= t} >= r, found bit by
//    bit from the top, each candidate counted per lane and summed over the warp.
// 2. Keep every J with key_J > T, and the (r - #{key_J > T}) lowest J with key_J == T.
template <int NPL, class KeyF, class EmitF>
__device__ __forceinline__ void warp_top_r(int n, int r, int lane, KeyF key_at, EmitF emit) {
  constexpr int kRegs = NPL > 0 ? NPL : 1;
  uint32_t o[kRegs];
  if constexpr (NPL > 0) {
#pragma unroll
    for (int k = 0; k < NPL; ++k) o[k] = (32 * k + lane < n) ? key_at(32 * k + lane) : 0u;
  }
  // Lanes past n are excluded from every count.
  auto count_ge = [&](uint32_t t) -> int {
    int c = 0;
    if constexpr (NPL > 0) {
#pragma unroll
      for (int k = 0; k < NPL; ++k) c += (32 * k + lane < n && o[k] >= t) ? 1 : 0;
    } else {
      for (int J = lane; J < n; J += 32) c += key_at(J) >= t ? 1 : 0;
    }
    return static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(c)));
  };
  uint32_t T = 0;
#pragma unroll 1
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cand = T | (1u << bit);
    if (count_ge(cand) >= r) T = cand;
  }
  const int n_gt = T == 0xFFFFFFFFu ? 0 : count_ge(T + 1u);
  const int n_eq_keep = r - n_gt;  // >= 1
  int base = 0, eq_seen = 0;
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int k = 0; 32 * k < n; ++k) {
    const int J = 32 * k + lane;
    uint32_t oj = 0;
    if constexpr (NPL > 0) {
#pragma unroll
      for (int kk = 0; kk < NPL; ++kk)
        if (kk == k) oj = o[kk];
    } else {
      oj = J < n ? key_at(J) : 0u;
    }
    const bool valid = J < n;
    const bool eq = valid && oj == T;
    const uint32_t m_eq = __ballot_sync(0xffffffffu, eq);
    const bool keep = valid && (oj > T || (eq && eq_seen + __popc(m_eq & lt_mask) < n_eq_keep));
    const uint32_t m = __ballot_sync(0xffffffffu, keep);
    if (keep) emit(J, base + __popc(m & lt_mask));
    base += __popc(m);
    eq_seen += __popc(m_eq);
  }
}

// Selection key of a score: NaN ranks last; -0 and +0 are one value (a tie, broken by J).
__device__ __forceinline__ uint32_t score_key(float v) {
  return ordered_bits(v != v ? -INFINITY : (v == 0.f ? 0.f : v));
}

// Top-r of the scores srow[0..nKB) written to out[0..r) in ascending J by one warp.
__device__ __forceinline__ void warp_top_r_scores(const float* srow, int nKB, int r, int lane, int32_t* out) {
  auto key = [&](int J) { return score_key(srow[J]); };
  auto emit = [&](int J, int pos) { out[pos] = J; };
  if (nKB <= 256) {
    warp_top_r<8>(nKB, r, lane, key, emit);
  } else if (nKB <= 512) {
    warp_top_r<16>(nKB, r, lane, key, emit);
  } else {
    warp_top_r<0>(nKB, r, lane, key, emit);
  }
}

// out[g * n + J] = q_sh[g] . rows[J] for the kSelQB query rows in shared memory and n fp32
// rows of D: a thread per row J, the row read with 16-byte loads, 8 in flight.
template <int D>
__device__ __forceinline__ void score_rows(const float (*q_sh)[D], const float* __restrict__ rows, int n,
                                           float* out) {
  for (int J = threadIdx.x; J < n; J += kSelectThreads) {
    const float4* krow = reinterpret_cast<const float4*>(rows + static_cast<size_t>(J) * D);
    float acc[kSelQB];
#pragma unroll
    for (int g = 0; g < kSelQB; ++g) acc[g] = 0.f;
#pragma unroll
    for (int k0 = 0; k0 < D / 4; k0 += 8) {
      float4 kv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) kv[u] = __ldg(krow + k0 + u);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
#pragma unroll
        for (int g = 0; g < kSelQB; ++g) {
          const float4 qv = *reinterpret_cast<const float4*>(&q_sh[g][4 * (k0 + u)]);
          acc[g] = fmaf(qv.x, kv[u].x, acc[g]);
          acc[g] = fmaf(qv.y, kv[u].y, acc[g]);
          acc[g] = fmaf(qv.z, kv[u].z, acc[g]);
          acc[g] = fmaf(qv.w, kv[u].w, acc[g]);
        }
      }
    }
#pragma unroll
    for (int g = 0; g < kSelQB; ++g) out[g * n + J] = acc[g];
  }
}

// idx_out[bh][I][0..r) = top-r key blocks of query block I, ascending.
// Scores: thread per key block J, s_IJ = Qbar_I . Kbar_J for the CTA's kSelQB query blocks
// (pooled Q in shared memory, the pooled K row streamed with 16-byte loads, all in flight).
// Selection: warp_top_r, one warp per query block.
template <int D>
__global__ void __launch_bounds__(kSelectThreads) score_select_kernel(const float* __restrict__ Qp,
                                                                      const float* __restrict__ Kp, int nQB,
                                                                      int nKB, int r,
                                                                      int32_t* __restrict__ idx_out,
                                                                      float* __restrict__ scores_out) {
  extern __shared__ float s_sc[];  // [kSelQB][nKB] scores
  __shared__ __align__(16) float q_sh[kSelQB][D];
  griddep_wait();
  griddep_launch_dependents();
  const int groups = (nQB + kSelQB - 1) / kSelQB;
  const int bh = blockIdx.x / groups;
  const int I0 = (blockIdx.x % groups) * kSelQB;
  const int G = min(kSelQB, nQB - I0);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  for (int i = threadIdx.x; i < kSelQB * D; i += kSelectThreads) {
    const int g = i / D;
    q_sh[g][i % D] = Qp[(static_cast<size_t>(bh) * nQB + I0 + min(g, G - 1)) * D + i % D];
  }
  __syncthreads();
  score_rows<D>(q_sh, Kp + static_cast<size_t>(bh) * nKB * D, nKB, s_sc);
  __syncthreads();

  if (warp < G) {
    const int I = I0 + warp;
    const float* srow = s_sc + warp * nKB;
    float* sout = scores_out ? scores_out + (static_cast<size_t>(bh) * nQB + I) * nKB : nullptr;
    if (sout)
      for (int J = lane; J < nKB; J += 32) sout[J] = srow[J];
    warp_top_r_scores(srow, nKB, r, lane, idx_out + (static_cast<size_t>(bh) * nQB + I) * r);
  }
}

// ------------------------------------------------------------ staged scoring
// score_select_staged_kernel: score_select_kernel with the head's pooled key means staged
// in shared memory, used when they fit (kStagedKBytes). The pooling kernel writes them
// transposed for it ([BH][D][nKB] fp32, contiguous per head), so that a few 32 KB bulk
// copies bring a head's means in at once, and thread J then reads column J: consecutive
// lanes read consecutive words (no bank conflicts) and every key block's dot products add
// over k in the same order, so equal key blocks give equal scores (the tie rule needs
// exact equality).
constexpr int kStagedKBytes = 192 * 1024;
constexpr int kStageCopyBytes = 32 * 1024;

template <int D>
__global__ void __launch_bounds__(kSelectThreads) score_select_staged_kernel(const float* __restrict__ Qp,
                                                                             const float* __restrict__ KpT, int nQB,
                                                                             int nKB, int r,
                                                                             int32_t* __restrict__ idx_out,
                                                                             float* __restrict__ scores_out,
                                                                             unsigned long long timeout_ns,
                                                                             int inject) {
  extern __shared__ __align__(128) float st_smem[];
  float* kcols = st_smem;                                // [D][nKB]
  float* s_sc = st_smem + static_cast<size_t>(nKB) * D;  // [kSelQB][nKB]
  __shared__ __align__(16) float q_sh[kSelQB][D];
  __shared__ uint64_t kbar;
  const int groups = (nQB + kSelQB - 1) / kSelQB;
  const int bh = blockIdx.x / groups;
  const int I0 = (blockIdx.x % groups) * kSelQB;
  const int G = min(kSelQB, nQB - I0);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t kbytes = static_cast<uint32_t>(nKB) * D * 4;  // a multiple of 16
  if (threadIdx.x == 0) {
    mbar_init(&kbar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  griddep_wait();
  griddep_launch_dependents();
  if (threadIdx.x == 0 && !inject) {  // test only: with inject the means never arrive
    const uint8_t* src = reinterpret_cast<const uint8_t*>(KpT + static_cast<size_t>(bh) * nKB * D);
    mbar_arrive_expect_tx(&kbar, kbytes);
    for (uint32_t o = 0; o < kbytes; o += kStageCopyBytes)
      bulk_load(reinterpret_cast<uint8_t*>(kcols) + o, src + o, min(kStageCopyBytes, static_cast<int>(kbytes - o)),
                &kbar);
  }
  for (int i = threadIdx.x; i < kSelQB * D; i += kSelectThreads) {
    const int g = i / D;
    q_sh[g][i % D] = Qp[(static_cast<size_t>(bh) * nQB + I0 + min(g, G - 1)) * D + i % D];
  }
  __syncthreads();
  // every thread waits for the means (the wait ignores the abort flag: issued copies must
  // land before the CTA exits)
  const bool landed = mbar_wait_drain(&kbar, 0, timeout_ns, (kKernSelect << 8) | 4);
  if (__syncthreads_or(!landed)) return;
  for (int J = threadIdx.x; J < nKB; J += kSelectThreads) {
    float acc[kSelQB];
#pragma unroll
    for (int g = 0; g < kSelQB; ++g) acc[g] = 0.f;
#pragma unroll 4
    for (int k0 = 0; k0 < D; k0 += 4) {
      float kv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) kv[u] = kcols[static_cast<size_t>(k0 + u) * nKB + J];
#pragma unroll
      for (int g = 0; g < kSelQB; ++g) {
        const float4 qv = *reinterpret_cast<const float4*>(&q_sh[g][k0]);
        acc[g] = fmaf(qv.x, kv[0], acc[g]);
        acc[g] = fmaf(qv.y, kv[1], acc[g]);
        acc[g] = fmaf(qv.z, kv[2], acc[g]);
        acc[g] = fmaf(qv.w, kv[3], acc[g]);
      }
    }
#pragma unroll
    for (int g = 0; g < kSelQB; ++g) s_sc[g * nKB + J] = acc[g];
  }
  __syncthreads();
  if (warp < G) {
    const int I = I0 + warp;
    const float* srow = s_sc + warp * nKB;
    float* sout = scores_out ? scores_out + (static_cast<size_t>(bh) * nQB + I) * nKB : nullptr;
    if (sout)
      for (int J = lane; J < nKB; J += 32) sout[J] = srow[J];
    warp_top_r_scores(srow, nKB, r, lane, idx_out + (static_cast<size_t>(bh) * nQB + I) * r);
  }
}

// ------------------------------------------------------------ pooled-key cache
// The window's keys as fp32 sums of G consecutive tokens ("granules"), in a ring of cap
// slots per (b, h): a chunk step sums only its new keys (kpool_push_kernel), and the
// selection pools its key blocks from the sums (kpool_blocks_kernel) instead of reading
// K. G divides the block size, so a key block is a whole run of granules.

// A push of n_new granules of G tokens of K ([BH][n_tokens][D]) into ring slots
// (base + g) % cap of sums ([BH][cap][D]).
struct PushArgs {
  const __nv_bfloat16* K;
  int n_tokens, G, n_new, base, cap;
  float* sums;
};

// sums[bh][(base + g) % cap][:] = sum of the rows [g*G, g*G + G) of K[bh], g < n_new, for
// the granules of push CTA `cta` (BH x ceil(n_new / granules per CTA) of them). A thread
// sums 8 columns of one granule (16-byte loads, 8 in flight); a warp reads whole rows (two
// granules at d = 128, four at d = 64).
template <int D>
__device__ __forceinline__ void push_granules(const PushArgs& q, int cta) {
  constexpr int kVec = 8;
  constexpr int kTpr = D / kVec;                 // threads per granule
  constexpr int kGran = kPoolThreads / kTpr;     // granules per CTA
  constexpr int kUnroll = 8;
  const int groups = (q.n_new + kGran - 1) / kGran;
  const int bh = cta / groups;
  const int g = (cta % groups) * kGran + threadIdx.x / kTpr;
  const int c = threadIdx.x % kTpr;
  if (g >= q.n_new) return;
  const __nv_bfloat16* X = q.K + (static_cast<size_t>(bh) * q.n_tokens + static_cast<size_t>(g) * q.G) * D + c * kVec;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  int row = 0;
  for (; row + kUnroll <= q.G; row += kUnroll) {
    uint4 v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) v[u] = ld_stream_16(X + static_cast<size_t>(row + u) * D);
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) acc_bf16x8(acc, v[u]);
  }
  for (; row < q.G; ++row) acc_bf16x8(acc, ld_stream_16(X + static_cast<size_t>(row) * D));
  float4* out =
      reinterpret_cast<float4*>(q.sums + (static_cast<size_t>(bh) * q.cap + (q.base + g) % q.cap) * D + c * kVec);
  out[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
  out[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
}

template <int D>
__global__ void __launch_bounds__(kPoolThreads) kpool_push_kernel(PushArgs q) {
  griddep_wait();
  griddep_launch_dependents();
  push_granules<D>(q, blockIdx.x);
}

// The query blocks' means (CTAs [0, BH nQB), as pool_blocks_kernel without key blocks) and
// a push (the other CTAs) in one launch: a chunk step's new keys enter the cache while its
// queries are pooled.
template <int D>
__global__ void __launch_bounds__(kPoolThreads, 8) pool_q_push_kernel(PoolArgs a, PushArgs q, int q_ctas) {
  __shared__ float red[PoolShape<D>::kRedFloats];
  griddep_wait();
  griddep_launch_dependents();
  if (static_cast<int>(blockIdx.x) < q_ctas)
    pool_block<D, false, false>(a, blockIdx.x / a.nQB, blockIdx.x % a.nQB, false, red, red);
  else
    push_granules<D>(q, blockIdx.x - q_ctas);
}

// Kp[bh][J][:] = mean of key block J of the window = (sum of its granule sums, in order) /
// its valid length; the window is the n_gran granules from ring slot head on. One warp per
// key block, D/32 columns a lane (512 contiguous bytes per load at d = 128), 8 in flight.
// kT: the means go out transposed, Kp[bh][k][J] (for score_select_staged_kernel): a CTA
// takes 8 consecutive key blocks of one (b, h), stages their means in shared memory and
// writes each k's 8 values as one 32-byte run.
template <int D, bool kT>
__global__ void __launch_bounds__(kPoolThreads) kpool_blocks_kernel(const float* __restrict__ sums, int cap,
                                                                    int head, int n_gran, int G, int block,
                                                                    int nKB, int BH, float* __restrict__ Kp) {
  constexpr int kC = D / 32;  // columns per lane: 4 or 2
  constexpr int kUnroll = 8;
  constexpr int kWarps = kPoolThreads / 32;
  __shared__ float tile[kT ? kWarps : 1][D];
  griddep_wait();
  griddep_launch_dependents();
  const int lane = threadIdx.x % 32, w = threadIdx.x / 32;
  int bh, J;
  if constexpr (kT) {
    const int groups = (nKB + kWarps - 1) / kWarps;
    bh = blockIdx.x / groups;
    J = (blockIdx.x % groups) * kWarps + w;
  } else {
    const long long wid = static_cast<long long>(blockIdx.x) * kWarps + w;
    if (wid >= static_cast<long long>(BH) * nKB) return;
    bh = static_cast<int>(wid / nKB);
    J = static_cast<int>(wid % nKB);
  }
  float acc[kC];
#pragma unroll
  for (int k = 0; k < kC; ++k) acc[k] = 0.f;
  const int per_block = block / G;
  const int g_lo = J * per_block, g_hi = min(g_lo + per_block, n_gran);
  if (J < nKB) {
    const float* S = sums + static_cast<size_t>(bh) * cap * D + lane * kC;
    for (int g0 = g_lo; g0 < g_hi; g0 += kUnroll) {
      float v[kUnroll][kC];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int g = g0 + u;
        if (g < g_hi) {
          const float* src = S + static_cast<size_t>((head + g) % cap) * D;
          if constexpr (kC == 4) {
            const float4 f = __ldg(reinterpret_cast<const float4*>(src));
            v[u][0] = f.x; v[u][1] = f.y; v[u][2] = f.z; v[u][3] = f.w;
          } else {
            const float2 f = __ldg(reinterpret_cast<const float2*>(src));
            v[u][0] = f.x; v[u][1] = f.y;
          }
        } else {
#pragma unroll
          for (int k = 0; k < kC; ++k) v[u][k] = 0.f;
        }
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
#pragma unroll
        for (int k = 0; k < kC; ++k) acc[k] += v[u][k];
      }
    }
  }
  const float L = static_cast<float>((g_hi - g_lo) * G);
  if constexpr (kT) {
    if (J < nKB) {
#pragma unroll
      for (int k = 0; k < kC; ++k) tile[w][lane * kC + k] = acc[k] / L;
    }
    __syncthreads();
    // thread t writes key block J0 + t % 8 of dimension t / 8 (+ 32 per step)
    const int j = threadIdx.x % kWarps, J0 = J - w;
    if (J0 + j < nKB) {
#pragma unroll
      for (int k = threadIdx.x / kWarps; k < D; k += kPoolThreads / kWarps)
        Kp[(static_cast<size_t>(bh) * D + k) * nKB + J0 + j] = tile[j][k];
    }
  } else {
    float* out = Kp + (static_cast<size_t>(bh) * nKB + J) * D + lane * kC;
#pragma unroll
    for (int k = 0; k < kC; ++k) out[k] = acc[k] / L;
  }
}

// ------------------------------------------------------------ two-stage selection
constexpr int kMaxKeyBlocks2 = 4096;  // block and frame scores of 4 query blocks in shared memory

template <int NPLMAX, class KeyF, class EmitF>
__device__ __forceinline__ void warp_top_r_dispatch(int n, int r, int lane, KeyF key, EmitF emit) {
  if (n <= 256) {
    warp_top_r<8>(n, r, lane, key, emit);
  } else if (NPLMAX >= 16 && n <= 512) {
    warp_top_r<16>(n, r, lane, key, emit);
  } else {
    warp_top_r<0>(n, r, lane, key, emit);
  }
}

// Source: "Light Forcing: Accelerating Autoregressive Video Diffusion via Sparse
// Attention", German technical summary, section 2.2 (two-stage mask selection: for each
// query block a small set of frames by the frame-level compressed keys, then the blocks
// within those frames by the block-level compressed keys).
// One CTA per (b, h, 4 query blocks): block scores s and frame scores f (a thread per
// row), then one warp per query block: the nf frames of largest f (ties to the lower
// frame; frames_out, ascending), candidate blocks = blocks with a token in a kept frame,
// and the r candidates of largest s (ties to the lower J) in ascending J. With fewer than
// r candidates every candidate is kept and the rest are the best other blocks.
// Dynamic shared memory: s[4][nKB], f[4][W] (fp32), kept[4][W], sel[4][nKB] (bytes).
template <int D>
__global__ void __launch_bounds__(kSelectThreads) score_select2_kernel(
    const float* __restrict__ Qp, const float* __restrict__ Kp, const float* __restrict__ Kf, int nQB, int nKB,
    int W, int Nk, int block, int T, int r, int nf, int32_t* __restrict__ idx_out, int32_t* __restrict__ frames_out,
    float* __restrict__ scores_out) {
  extern __shared__ float dsm[];
  float* s_sc = dsm;
  float* f_sc = s_sc + kSelQB * nKB;
  uint8_t* kept = reinterpret_cast<uint8_t*>(f_sc + kSelQB * W);
  uint8_t* sel = kept + kSelQB * W;
  __shared__ __align__(16) float q_sh[kSelQB][D];
  griddep_wait();
  griddep_launch_dependents();
  const int groups = (nQB + kSelQB - 1) / kSelQB;
  const int bh = blockIdx.x / groups;
  const int I0 = (blockIdx.x % groups) * kSelQB;
  const int G = min(kSelQB, nQB - I0);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  for (int i = threadIdx.x; i < kSelQB * D; i += kSelectThreads) {
    const int g = i / D;
    q_sh[g][i % D] = Qp[(static_cast<size_t>(bh) * nQB + I0 + min(g, G - 1)) * D + i % D];
  }
  __syncthreads();
  score_rows<D>(q_sh, Kp + static_cast<size_t>(bh) * nKB * D, nKB, s_sc);
  score_rows<D>(q_sh, Kf + static_cast<size_t>(bh) * W * D, W, f_sc);
  __syncthreads();

  if (warp < G) {
    const int I = I0 + warp;
    const size_t q = static_cast<size_t>(bh) * nQB + I;
    const float* srow = s_sc + warp * nKB;
    const float* frow = f_sc + warp * W;
    uint8_t* krow = kept + warp * W;
    uint8_t* selrow = sel + warp * nKB;
    if (scores_out)
      for (int J = lane; J < nKB; J += 32) scores_out[q * nKB + J] = srow[J];
    for (int w = lane; w < W; w += 32) krow[w] = 0;
    __syncwarp();
    // stage 1: the nf frames of largest score
    int32_t* fout = frames_out ? frames_out + q * nf : nullptr;
    warp_top_r_dispatch<8>(
        W, nf, lane, [&](int w) { return score_key(frow[w]); },
        [&](int w, int pos) {
          krow[w] = 1;
          if (fout) fout[pos] = w;
        });
    __syncwarp();
    // stage 2: candidate blocks (a token in a kept frame; a block touches at most 2 frames)
    auto is_cand = [&](int J) -> bool {
      const int f_lo = (J * block) / T;
      const int f_hi = (min((J + 1) * block, Nk) - 1) / T;
      return (krow[f_lo] | krow[f_hi]) != 0;
    };
    int nc = 0;
    for (int J = lane; J < nKB; J += 32) nc += is_cand(J) ? 1 : 0;
    nc = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(nc)));
    int32_t* out = idx_out + q * r;
    if (nc >= r) {
      warp_top_r_dispatch<16>(
          nKB, r, lane, [&](int J) { return is_cand(J) ? score_key(srow[J]) : 0u; },
          [&](int J, int pos) { out[pos] = J; });
    } else {
      // every candidate, then the best r - nc other blocks; written in ascending J
      for (int J = lane; J < nKB; J += 32) selrow[J] = is_cand(J) ? 1 : 0;
      __syncwarp();
      warp_top_r_dispatch<16>(
          nKB, r - nc, lane, [&](int J) { return is_cand(J) ? 0u : score_key(srow[J]); },
          [&](int J, int) { selrow[J] = 1; });
      __syncwarp();
      int base = 0;
      const uint32_t lt_mask = (1u << lane) - 1u;
      for (int J0 = 0; J0 < nKB; J0 += 32) {
        const int J = J0 + lane;
        const bool keep = J < nKB && selrow[J] != 0;
        const uint32_t m = __ballot_sync(0xffffffffu, keep);
        if (keep) out[base + __popc(m & lt_mask)] = J;
        base += __popc(m);
      }
    }
  }
}

}  // namespace hf

// Block scoring and top-r selection (hf_select_blocks).
//
// Source: "Light Forcing: Accelerating Autoregressive Video Diffusion via Sparse
// Attention", German technical summary, section 2.2 (query and key tokens are
// compressed by mean pooling at block level; key blocks are selected per query
// block); "Long-Horizon Streaming Video Generation via Hybrid Attention with
// Decoupled Distillation", German technical summary, section 2 A (only the most
// important, Top-K, blocks are computed).
//
// Two kernels, both on CUDA cores (the work is a streaming read of Q and K plus a
// tiny score matrix, so tensor cores would not help):
//   pool_blocks_kernel   one CTA per (b,h,block) of Q or K: fp32 mean of the valid rows.
//                        HBM-bound: reads Q and K once with 16-byte loads, 8 in flight
//                        per thread.
//   score_select_kernel  one CTA per (b,h, 4 query blocks): s_IJ = Qbar_I . Kbar_J, a
//                        thread per key block; then one warp per query block finds the
//                        r-th largest score by a bitwise search (per-lane counts, one warp
//                        reduction per bit), takes every block above it and the lowest-J
//                        blocks equal to it, and writes the r blocks in ascending J.
//                        NaN scores are ranked as -inf, so exactly r blocks are written.
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

// Qp[bh][I][:] = mean of Q rows of block I; Kp[bh][J][:] likewise.
template <int D>
__global__ void __launch_bounds__(kPoolThreads) pool_blocks_kernel(const __nv_bfloat16* __restrict__ Q,
                                                                   const __nv_bfloat16* __restrict__ K,
                                                                   int Nq, int Nk, int block, int nQB, int nKB,
                                                                   float* __restrict__ Qp,
                                                                   float* __restrict__ Kp) {
  constexpr int kVec = 8;                       // bf16 per 16-byte load
  constexpr int kTpr = D / kVec;                // threads per row
  constexpr int kRows = kPoolThreads / kTpr;    // rows per pass
  constexpr int kUnroll = 8;                    // loads in flight per thread
  __shared__ float red[kRows * D];

  const int per_bh = nQB + nKB;
  const int bh = blockIdx.x / per_bh;
  int t = blockIdx.x % per_bh;
  const __nv_bfloat16* X;
  int N;
  float* out;
  if (t < nQB) {
    X = Q + static_cast<size_t>(bh) * Nq * D;
    N = Nq;
    out = Qp + (static_cast<size_t>(bh) * nQB + t) * D;
  } else {
    t -= nQB;
    X = K + static_cast<size_t>(bh) * Nk * D;
    N = Nk;
    out = Kp + (static_cast<size_t>(bh) * nKB + t) * D;
  }
  const int lo = t * block;
  const int hi = min(lo + block, N);
  const int c = threadIdx.x % kTpr;
  const int rr = threadIdx.x / kTpr;

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
#pragma unroll
  for (int k = 0; k < 8; ++k) red[rr * D + c * kVec + k] = acc[k];
  __syncthreads();
  if (threadIdx.x < D) {
    float s = 0.f;
#pragma unroll 8
    for (int q = 0; q < kRows; ++q) s += red[q * D + threadIdx.x];
    out[threadIdx.x] = s / static_cast<float>(hi - lo);
  }
}

// Scores of kSelQB query blocks of one head per CTA (each pooled K row is read once for
// all of them), then one warp per query block selects its top r.
constexpr int kSelQB = 4;

// Order-preserving map of a float to an unsigned integer (NaN has been replaced by -inf).
__device__ __forceinline__ uint32_t ordered_bits(float f) {
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Top-r of the scores srow[0..nKB) (larger score first, lower J first on ties), written
// to out[0..r) in ascending J by one warp. NPL = ordered scores per lane held in registers
// (lane l holds J = 32 k + l); NPL = 0 reads shared memory each time (any nKB).
// 1. T = the r-th largest ordered score: the largest t with #{J : o_J >= t} >= r, found
//    bit by bit from the top, each candidate counted per lane and summed over the warp.
// 2. Keep every J with o_J > T, and the (r - #{o_J > T}) lowest J with o_J == T.
template <int NPL>
__device__ __forceinline__ void warp_top_r(const float* srow, int nKB, int r, int lane, int32_t* out) {
  auto ob_at = [&](int J) -> uint32_t {
    const float v = srow[J];
    // NaN ranks last; -0 and +0 are one value (a tie, broken by J)
    return ordered_bits(v != v ? -INFINITY : (v == 0.f ? 0.f : v));
  };
  constexpr int kRegs = NPL > 0 ? NPL : 1;
  uint32_t o[kRegs];
  if constexpr (NPL > 0) {
#pragma unroll
    for (int k = 0; k < NPL; ++k) o[k] = (32 * k + lane < nKB) ? ob_at(32 * k + lane) : 0u;
  }
  // Lanes past nKB are excluded from every count (their register holds 0).
  auto count_ge = [&](uint32_t t) -> int {
    int c = 0;
    if constexpr (NPL > 0) {
#pragma unroll
      for (int k = 0; k < NPL; ++k) c += (32 * k + lane < nKB && o[k] >= t) ? 1 : 0;
    } else {
      for (int J = lane; J < nKB; J += 32) c += ob_at(J) >= t ? 1 : 0;
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
  for (int k = 0; 32 * k < nKB; ++k) {
    const int J = 32 * k + lane;
    uint32_t oj = 0;
    if constexpr (NPL > 0) {
#pragma unroll
      for (int kk = 0; kk < NPL; ++kk)
        if (kk == k) oj = o[kk];
    } else {
      oj = J < nKB ? ob_at(J) : 0u;
    }
    const bool valid = J < nKB;
    const bool eq = valid && oj == T;
    const uint32_t m_eq = __ballot_sync(0xffffffffu, eq);
    const bool keep = valid && (oj > T || (eq && eq_seen + __popc(m_eq & lt_mask) < n_eq_keep));
    const uint32_t m = __ballot_sync(0xffffffffu, keep);
    const int pos = base + __popc(m & lt_mask);
    if (keep) out[pos] = J;
    base += __popc(m);
    eq_seen += __popc(m_eq);
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
  const float* kbase = Kp + static_cast<size_t>(bh) * nKB * D;
  for (int J = threadIdx.x; J < nKB; J += kSelectThreads) {
    const float4* krow = reinterpret_cast<const float4*>(kbase + static_cast<size_t>(J) * D);
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
    for (int g = 0; g < kSelQB; ++g) s_sc[g * nKB + J] = acc[g];
  }
  __syncthreads();

  if (warp < G) {
    const int I = I0 + warp;
    const float* srow = s_sc + warp * nKB;
    float* sout = scores_out ? scores_out + (static_cast<size_t>(bh) * nQB + I) * nKB : nullptr;
    if (sout)
      for (int J = lane; J < nKB; J += 32) sout[J] = srow[J];
    int32_t* out = idx_out + (static_cast<size_t>(bh) * nQB + I) * r;
    if (nKB <= 256) {
      warp_top_r<8>(srow, nKB, r, lane, out);
    } else if (nKB <= 512) {
      warp_top_r<16>(srow, nKB, r, lane, out);
    } else {
      warp_top_r<0>(srow, nKB, r, lane, out);
    }
  }
}

}  // namespace hf

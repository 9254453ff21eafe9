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
//   score_select_kernel  one CTA per (b,h,I): s_IJ = Qbar_I . Kbar_J by warp-level
//                        reductions (one warp per J, lanes over d, xor shuffles), then
//                        rank_J = #{J': s_J' > s_J or (s_J' == s_J and J' < J)}; the
//                        r blocks with rank < r are written in ascending J. NaN scores
//                        are ranked as -inf so exactly r blocks are always written.
#pragma once

#include "hf_ptx.cuh"

namespace hf {

constexpr int kPoolThreads = 256;
constexpr int kSelectThreads = 256;
constexpr int kMaxKeyBlocks = 8192;  // score row + flags fit in shared memory

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

// idx_out[bh][I][0..r) = top-r key blocks of query block I, ascending.
template <int D>
__global__ void __launch_bounds__(kSelectThreads) score_select_kernel(const float* __restrict__ Qp,
                                                                      const float* __restrict__ Kp, int nQB,
                                                                      int nKB, int r,
                                                                      int32_t* __restrict__ idx_out,
                                                                      float* __restrict__ scores_out) {
  extern __shared__ float s_row[];  // [nKB] scores, then [nKB] int flags
  int* flag = reinterpret_cast<int*>(s_row + nKB);
  constexpr int kPer = D / 32;  // pooled elements per lane
  const int bh = blockIdx.x / nQB;
  const int I = blockIdx.x % nQB;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  constexpr int kWarps = kSelectThreads / 32;

  float q[kPer];
  const float* qrow = Qp + (static_cast<size_t>(bh) * nQB + I) * D + lane * kPer;
#pragma unroll
  for (int k = 0; k < kPer; ++k) q[k] = qrow[k];

  const float* kbase = Kp + static_cast<size_t>(bh) * nKB * D + lane * kPer;
  for (int J = warp; J < nKB; J += kWarps) {
    const float* krow = kbase + static_cast<size_t>(J) * D;
    float dot = 0.f;
#pragma unroll
    for (int k = 0; k < kPer; ++k) dot = fmaf(q[k], krow[k], dot);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
    if (lane == 0) s_row[J] = dot;
  }
  __syncthreads();

  float* srow_out = scores_out ? scores_out + (static_cast<size_t>(bh) * nQB + I) * nKB : nullptr;
  for (int J = threadIdx.x; J < nKB; J += kSelectThreads) {
    const float v = s_row[J];
    if (srow_out) srow_out[J] = v;
  }
  __syncthreads();
  // NaN ranks last; the order (score desc, index asc) is then a strict total order.
  for (int J = threadIdx.x; J < nKB; J += kSelectThreads) {
    if (s_row[J] != s_row[J]) s_row[J] = -INFINITY;
  }
  __syncthreads();

  for (int J = threadIdx.x; J < nKB; J += kSelectThreads) {
    const float v = s_row[J];
    int rank = 0;
    for (int Jp = 0; Jp < nKB; ++Jp) {
      const float w = s_row[Jp];
      rank += (w > v) || (w == v && Jp < J);
    }
    flag[J] = rank < r;
  }
  __syncthreads();

  int32_t* out = idx_out + (static_cast<size_t>(bh) * nQB + I) * r;
  for (int J = threadIdx.x; J < nKB; J += kSelectThreads) {
    if (!flag[J]) continue;
    int pos = 0;
    for (int Jp = 0; Jp < J; ++Jp) pos += flag[Jp];
    if (pos < r) out[pos] = J;
  }
}

}  // namespace hf

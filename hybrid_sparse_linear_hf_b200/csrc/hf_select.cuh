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
//                        thread per key block; then one warp per query block finds its
//                        top r by a warp-wide bitwise search (ballots) for the r-th
//                        largest (score, -J) key; the r blocks are written in ascending J.
//                        NaN scores are ranked as -inf, so exactly r blocks are written.
#pragma once

#include "hf_ptx.cuh"

namespace hf {

constexpr int kPoolThreads = 256;
constexpr int kSelectThreads = 256;
constexpr int kMaxKeyBlocks = 8192;  // 4 score rows fit in shared memory; J fits the 13-bit key field

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
constexpr int kSelRegKeys = 16;  // keys per lane held in registers (nKB <= 512)

// Order-preserving map of a float to an unsigned integer (NaN has been replaced by -inf).
__device__ __forceinline__ uint32_t ordered_bits(float f) {
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Unique selection key of key block J: larger score first, lower index first on ties.
__device__ __forceinline__ uint64_t select_key(float s, int J) {
  return (static_cast<uint64_t>(ordered_bits(s)) << 13) | static_cast<uint64_t>(8191 - J);
}

// idx_out[bh][I][0..r) = top-r key blocks of query block I, ascending.
// Scores: thread per key block J, s_IJ = Qbar_I . Kbar_J for the CTA's kSelQB query blocks
// (pooled Q in shared memory, the pooled K row streamed with 16-byte loads, all in flight).
// Selection: the warp of query block I finds the r-th largest of the unique 45-bit keys
// (ordered score bits << 13) | (8191 - J) bit by bit (counting keys at or above a
// candidate with ballots); the blocks at or above it are exactly the top r, written in
// ascending J with ballot prefix counts.
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
    auto key_at = [&](int J) -> uint64_t {
      const float v = srow[J];
      return select_key(v != v ? -INFINITY : v, J);  // NaN ranks last
    };
    // largest T with #{keys >= T} >= r: the r-th largest key (keys are unique)
    uint64_t T = 0;
    if (nKB <= 32 * kSelRegKeys) {
      uint64_t keys[kSelRegKeys];
#pragma unroll
      for (int k = 0; k < kSelRegKeys; ++k) keys[k] = (32 * k + lane < nKB) ? key_at(32 * k + lane) : 0ull;
      for (int bit = 44; bit >= 0; --bit) {
        const uint64_t cand = T | (1ull << bit);
        int cnt = 0;
#pragma unroll
        for (int k = 0; k < kSelRegKeys; ++k) cnt += __popc(__ballot_sync(0xffffffffu, keys[k] >= cand));
        if (cnt >= r) T = cand;
      }
    } else {
      for (int bit = 44; bit >= 0; --bit) {
        const uint64_t cand = T | (1ull << bit);
        int cnt = 0;
        for (int J0 = 0; J0 < nKB; J0 += 32) {
          const int J = J0 + lane;
          cnt += __popc(__ballot_sync(0xffffffffu, J < nKB && key_at(J) >= cand));
        }
        if (cnt >= r) T = cand;
      }
    }
    int32_t* out = idx_out + (static_cast<size_t>(bh) * nQB + I) * r;
    int base = 0;
    for (int J0 = 0; J0 < nKB; J0 += 32) {
      const int J = J0 + lane;
      const bool keep = J < nKB && key_at(J) >= T;
      const uint32_t m = __ballot_sync(0xffffffffu, keep);
      const int pos = base + __popc(m & ((1u << lane) - 1u));
      if (keep && pos < r) out[pos] = J;
      base += __popc(m);
    }
  }
}

}  // namespace hf

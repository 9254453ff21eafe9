// State absorption (hf_absorb_evicted): S += phi(K)^T V, z += sum_t phi(k_t).
//
// Source: "Long-Horizon Streaming Video Generation via Hybrid Attention with
// Decoupled Distillation", German technical summary, section 2 A (frames evicted
// from the sliding window are aggregated into a compact KV state through a linear
// attention function, constant memory in the video length); English abstract
// (a compact key-value state incrementally absorbs evicted tokens).
//
// Work split: the tokens of every (b,h) are cut into `nsplit` slices of whole
// 64-token tiles; one CTA per (b,h,slice) accumulates its slice's phi(K)^T V and writes
// an fp32 partial; reduce_state_kernel adds the partials of a head to S and z in slice
// order (deterministic).
//
// absorb_partial_kernel (576 threads, one CTA per SM). The product is computed transposed,
//   D[n][c] = sum_t V[t][n] * B[t][c],   B = [phi_hi | phi_lo]  (N = 2d columns),
// so that one MMA of M = 128 (n, zero-padded rows for d = 64), N = 2d, K = 16 tokens covers
// both halves of the split: S[k][n] = D[n][k] + D[n][d + k]. Both operands are MN-major
// (the element index contiguous): A = V^T is the V tile as TMA wrote it, B is the
// converted K tile.
//   warp 0      TMA producer: the V and K tiles [64 tokens][d] of a tile into one ring
//               stage laid out [V | K, then phi_hi over K | phi_lo], 64-column chunks of
//               8 KB each, so the A chunks and the 2d/64 B chunks are 8 KB apart.
//   warp 1      TMEM owner + MMA issuer: per tile 4 MMAs (K = 16 tokens each) into one of
//               two TMEM accumulators of 2d columns. It waits only for the converters'
//               "B written" barrier of the stage (they arrive after the stage barrier, so
//               the V tile has landed too) and commits the stage back to the producer.
//   warps 2..17 converters (four warps per SM sub-partition: the conversion is issue- and
//               MUFU-bound): phi(k) in fp32, split hi = bf16(phi), lo = bf16(phi - hi);
//               hi overwrites the K chunk in place and lo goes to the stage's lo chunk; z
//               is accumulated in fp32 registers. They also drain the accumulator: the
//               tensor core's fp32 accumulation truncates, so a long chain of MMAs into one
//               TMEM accumulator drifts (relative error grows with the chain length, ~2e-5
//               after 500 MMAs). The MMAs of every group of kAbsGroup tiles (512 tokens)
//               therefore go to one of two TMEM accumulators, which the converters add into
//               fp32 registers with round-to-nearest while the other one fills; the four
//               warps that share a TMEM lane quarter (rows n) take a quarter of the k
//               columns each, hi and lo halves together. Epilogue: registers -> fp32 partial
//               S[k][n] in the workspace.
// Rows past the end of the token range are zero-filled by TMA; their phi is forced to 0
// (phi(0) = 1 would otherwise leak into z).
// The converters arrive on the "B written" and "accumulator drained" barriers once per
// warp (after a __syncwarp), not once per thread: 16 arrivals per tile instead of 512.
// Launch order: with `wait_first` the kernel waits for the previous grid of its stream
// before its first load (its inputs may come from it); without, it reads K and V at once
// (the caller guarantees they were complete before the previous grid started) and waits
// only before it exits, so that the next grid of the stream sees the previous one done.
#pragma once

#include "hf_ptx.cuh"

namespace hf {

constexpr uint32_t kKernAbsorb = 2;
constexpr int kAbsTok = 64;        // tokens per tile
constexpr int kAbsMaxStages = 8;   // ring depth cap
constexpr int kConvThreads = 512;  // converter warps 2..17
constexpr int kAbsThreads = 64 + kConvThreads;
constexpr int kAbsGroup = 8;       // tiles per TMEM accumulation chain
constexpr int kConvGroups = 2;     // converter groups; group g converts the tiles i with i % 2 == g

template <int D>
struct AbsorbCfg {
  static constexpr int kChunks = D / 64;                  // 64-element column chunks of a tile
  static constexpr int kChunkBytes = kAbsTok * 128;       // one chunk: 64 rows x 128 B
  static constexpr int kTileBytes = kChunks * kChunkBytes;
  static constexpr int kStageBytes = 3 * kTileBytes;      // V | K (-> phi_hi) | phi_lo
  static constexpr int kVOff = 0;
  static constexpr int kKOff = kTileBytes;
  static constexpr int kLoOff = 2 * kTileBytes;
  static constexpr int kN = 2 * D;                        // MMA N: phi_hi and phi_lo columns
  static constexpr uint32_t kAccCols = kN;                // TMEM columns per accumulator
  static constexpr uint32_t kTmemCols = 2 * kAccCols;     // two accumulators (256 or 512)
  static constexpr int kZredBytes = kConvThreads * 8 * 4;  // end-of-kernel z reduction (over the ring)
  static constexpr int kBudget = 232448 - 1024 - 1024;    // shared memory per CTA - alignment - static
  static constexpr int kStagesFit = kBudget / kStageBytes;
  static constexpr int kStages = kStagesFit < kAbsMaxStages ? kStagesFit : kAbsMaxStages;
  static_assert(kStages >= 2, "ring too small");
  static constexpr int kRingBytes = kStages * kStageBytes;
  static_assert(kZredBytes <= kRingBytes, "z reduction must fit over the ring");
  static constexpr int kDynSmem = 1024 + kRingBytes;
  static constexpr int kColsPerWarp = D / 4;              // k columns per converter warp in the drain
  static_assert(kTmemCols == 256 || kTmemCols == 512, "TMEM allocation is a power of two");
};

struct AbsorbParams {
  float* part_S;  // [BH][nsplit][D][D]
  float* part_z;  // [BH][nsplit][D]
  int n_tokens;   // tokens per (b,h)
  int tiles_per_split;
  int nsplit;
  int wait_first;  // 1: wait for the previous grid before the first load
  unsigned long long timeout_ns;
  int inject;     // test only: skip the first tile's load so a wait runs out
};

template <int D>
__global__ void __launch_bounds__(kAbsThreads, 1)
    absorb_partial_kernel(const __grid_constant__ CUtensorMap mapK, const __grid_constant__ CUtensorMap mapV,
                          AbsorbParams p) {
  using C = AbsorbCfg<D>;
  constexpr int NS = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  __shared__ uint64_t full_bar[NS], empty_bar[NS], bfull_bar[NS];
  __shared__ uint64_t dfull_bar[2], dempty_bar[2], drain_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int bh = blockIdx.x / p.nsplit;
  const int split = blockIdx.x % p.nsplit;
  const int tile0 = split * p.tiles_per_split;
  const int tiles_total = (p.n_tokens + kAbsTok - 1) / kAbsTok;
  const int ntiles = min(p.tiles_per_split, tiles_total - tile0);
  volatile int* abort_flag = &abort_sh;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
      mbar_init(&bfull_bar[s], kConvThreads / 32 / kConvGroups);  // the converting group's warps
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&dfull_bar[b], 1);
      mbar_init(&dempty_bar[b], kConvThreads / 32);
    }
    mbar_init(&drain_bar, 1);
    abort_sh = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&mapK);
    tma_prefetch_desc(&mapV);
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = tmem_base_sh;
  // the next kernel of the stream (the slice reduction) may be scheduled now
  griddep_launch_dependents();

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      if (p.wait_first) griddep_wait();
      int issued = 0;
      for (int i = 0; i < ntiles; ++i) {
        const int s = i % NS, u = i / NS;
        if (u >= 1 && !mbar_wait(&empty_bar[s], (u - 1) & 1, abort_flag, p.timeout_ns, (kKernAbsorb << 8) | 1))
          break;
        if (*abort_flag) break;
        if (p.inject && i == 0) continue;  // test only: tile 0 never arrives
        uint8_t* st = ring + s * C::kStageBytes;
        mbar_arrive_expect_tx(&full_bar[s], 2 * C::kTileBytes);
        const int row = (tile0 + i) * kAbsTok;
#pragma unroll
        for (int c = 0; c < C::kChunks; ++c) {
          tma_load_3d(st + C::kVOff + c * C::kChunkBytes, &mapV, &full_bar[s], c * 64, row, bh);
          tma_load_3d(st + C::kKOff + c * C::kChunkBytes, &mapK, &full_bar[s], c * 64, row, bh);
        }
        issued = i + 1;
      }
      // drain: every issued copy must have landed before the CTA may exit
      for (int i = max(0, issued - NS); i < issued; ++i) {
        if (p.inject && i == 0) continue;
        mbar_wait_drain(&full_bar[i % NS], (i / NS) & 1, p.timeout_ns, (kKernAbsorb << 8) | 2);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      // A = V^T (M = 128: the d columns of V, MN-major; for d = 64 the second M chunk is
      // the next 8 KB of the stage, whose products land in TMEM rows that are never read),
      // B = [phi_hi | phi_lo] (N = 2d, MN-major); chunks 8 KB apart, 8-row groups 1 KB apart
      constexpr uint32_t idesc = idesc_bf16_f32(128, C::kN, true, true);
      const uint64_t adesc0 = sdesc_sw128(smem_u32(ring + C::kVOff), C::kChunkBytes, 1024);
      const uint64_t bdesc0 = sdesc_sw128(smem_u32(ring + C::kKOff), C::kChunkBytes, 1024);
      bool ok = true;
      for (int i = 0; i < ntiles && ok; ++i) {
        const int s = i % NS;
        const int g = i / kAbsGroup, b = g & 1;
        const bool first = (i % kAbsGroup) == 0;
        const bool last = (i % kAbsGroup) == kAbsGroup - 1 || i == ntiles - 1;
        ok = mbar_wait(&bfull_bar[s], (i / NS) & 1, abort_flag, p.timeout_ns, (kKernAbsorb << 8) | 4);
        if (ok && first && g >= 2)
          ok = mbar_wait(&dempty_bar[b], ((g >> 1) - 1) & 1, abort_flag, p.timeout_ns, (kKernAbsorb << 8) | 9);
        if (!ok) break;
        tc_fence_after();
        const uint64_t so = static_cast<uint64_t>((s * C::kStageBytes) >> 4);
        const uint32_t d_tmem = tmem_d + b * C::kAccCols;
#pragma unroll
        for (int ks = 0; ks < kAbsTok / 16; ++ks)  // 16 tokens = 16 rows of 128 B = 2048 B
          umma_ss(d_tmem, adesc0 + so + ks * 128, bdesc0 + so + ks * 128, idesc, (!first || ks > 0) ? 1u : 0u);
        umma_commit(&empty_bar[s]);
        if (last) umma_commit(&dfull_bar[b]);
      }
      umma_commit(&drain_bar);
      mbar_wait_drain(&drain_bar, 0, p.timeout_ns, (kKernAbsorb << 8) | 5);
    }
  } else {
    // ---------------- converters + epilogue (512 threads) ----------------
    const int t = threadIdx.x - 64;
    constexpr int kUnits = D / 8;    // 16-byte units per row
    constexpr int kPhases = kConvThreads / kUnits;  // (over both groups, for the z reduction)
    constexpr int kGroupThreads = kConvThreads / kConvGroups;
    constexpr int kGPhases = kGroupThreads / kUnits;
    constexpr int kRowsPerThread = kAbsTok / kGPhases;
    static_assert(kGPhases % 8 == 0, "a thread's rows share their swizzle phase");
    // each ring stage serves one group only, so a group waits on a stage's phases in order
    static_assert(NS % kConvGroups == 0, "ring stages per converter group");
    // The two groups convert alternate tiles, so that one group's arithmetic overlaps the
    // other's waits and the tile stream; all converter warps drain the accumulators.
    const int cgroup = t / kGroupThreads;
    const int ucol = t % kUnits;     // logical unit column: elements [8*ucol, 8*ucol + 8)
    const int phase = (t % kGroupThreads) / kUnits;  // rows phase, phase + kGPhases, ...
    const int chunk = ucol / 8;
    const uint32_t swz = static_cast<uint32_t>(((ucol % 8) ^ (phase & 7)) * 16);
    uint64_t zacc[4] = {0ull, 0ull, 0ull, 0ull};  // fp32 pairs: elements (2e, 2e+1) of the unit
    // register accumulator: row n of D (TMEM lane n), k columns [col0, col0 + NC) of both
    // halves; the four warps that share a TMEM lane quarter (warp % 4) take a quarter each
    constexpr int NC = C::kColsPerWarp;
    const int quarter = warp & 3;
    const int n_row = quarter * 32 + lane;
    const bool drains = n_row < D;  // for d = 64 lanes 64..127 hold padding rows (warp-uniform)
    const int col0 = ((warp - 2) / 4) * NC;
    const uint32_t lane_base = tmem_d + (static_cast<uint32_t>(quarter * 32) << 16);
    float acc[NC];
#pragma unroll
    for (int c = 0; c < NC; ++c) acc[c] = 0.f;
    const int ngroups = (ntiles + kAbsGroup - 1) / kAbsGroup;
    int flushed = 0;
    bool ok = true;
    auto flush_group = [&](int g) {
      const int b = g & 1;
      // the TMEM loads below are warp-collective: the wait result is made warp-uniform
      if (!__all_sync(0xffffffffu,
                      mbar_wait(&dfull_bar[b], (g >> 1) & 1, abort_flag, p.timeout_ns, (kKernAbsorb << 8) | 8)))
        return false;
      tc_fence_after();
      if (drains) {
        // the hi half, then the lo half (one half in registers at a time)
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t r[NC];
          tmem_ld_cols<NC>(lane_base + b * C::kAccCols + half * D + col0, r);
          tmem_wait_ld();
          reg_fence<NC>(r);
#pragma unroll
          for (int j = 0; j < NC; ++j) acc[j] += __uint_as_float(r[j]);
        }
      }
      // one arrival per warp once all its lanes' TMEM loads are done
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&dempty_bar[b]);
      return true;
    };
    // phi(x) = x + 1 (x > 0) or exp(x) (x <= 0) for the two bf16 halves of w, in fp32,
    // written branch-free as (x - m) + 2^(m log2 e) with m = min(x, 0) (the exponential
    // is 1 for x > 0; x - m, exact, is one packed FMA instead of two max operations on
    // the busier ALU pipe); hi = bf16(phi), lo = bf16(phi - hi); z accumulates phi.
    auto convert_pair = [&](uint32_t w, uint64_t& z2, uint32_t& hi, uint32_t& lo) {
      const float x0 = bf16_lo_to_f32(w), x1 = bf16_hi_to_f32(w);
      const uint64_t m2 = f32x2(fminf(x0, 0.f), fminf(x1, 0.f));
      float l0, l1;
      f32x2_split(ffma2(m2, f32x2(1.4426950408889634f, 1.4426950408889634f), 0ull), l0, l1);
      const uint64_t xm = ffma2(m2, f32x2(-1.0f, -1.0f), f32x2(x0, x1));
      const uint64_t pp = fadd2(xm, f32x2(ex2_approx(l0), ex2_approx(l1)));
      float p0, p1;
      f32x2_split(pp, p0, p1);
      z2 = fadd2(z2, pp);
      hi = pack_bf16x2(p0, p1);
      float r0, r1;
      f32x2_split(ffma2(f32x2(bf16_lo_to_f32(hi), bf16_hi_to_f32(hi)), f32x2(-1.0f, -1.0f), pp), r0, r1);
      lo = pack_bf16x2(r0, r1);
    };
    for (int i = cgroup; i < ntiles && ok; i += kConvGroups) {
      const int s = i % NS;
      ok = __all_sync(0xffffffffu,
                      mbar_wait(&full_bar[s], (i / NS) & 1, abort_flag, p.timeout_ns, (kKernAbsorb << 8) | 6));
      if (!ok) break;
      uint8_t* stage = ring + s * C::kStageBytes;
      const int valid = min(kAbsTok, p.n_tokens - (tile0 + i) * kAbsTok);
#pragma unroll
      for (int k = 0; k < kRowsPerThread; ++k) {
        const int row = phase + k * kGPhases;
        const uint32_t off = chunk * C::kChunkBytes + row * 128 + swz;
        const uint4 kv = *reinterpret_cast<const uint4*>(stage + C::kKOff + off);
        uint32_t hi[4], lo[4];
        if (valid == kAbsTok || row < valid) {
          convert_pair(kv.x, zacc[0], hi[0], lo[0]);
          convert_pair(kv.y, zacc[1], hi[1], lo[1]);
          convert_pair(kv.z, zacc[2], hi[2], lo[2]);
          convert_pair(kv.w, zacc[3], hi[3], lo[3]);
        } else {
          // rows past the end of the tokens (zero-filled by TMA): phi forced to 0
#pragma unroll
          for (int e = 0; e < 4; ++e) hi[e] = lo[e] = 0u;
        }
        *reinterpret_cast<uint4*>(stage + C::kKOff + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(stage + C::kLoOff + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
      // every lane's stores are made visible to the tensor core, then one arrival per warp
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bfull_bar[s]);
      // once this thread's share of group g is converted, drain group g - 1 (one group of lag
      // keeps the tensor core busy on the other accumulator)
      const int g = i / kAbsGroup;
      const bool group_done = (i + kConvGroups) / kAbsGroup != g || i + kConvGroups >= ntiles;
      if (group_done && g >= 1) {
        ok = flush_group(g - 1);
        flushed = g;
      }
    }
    if (ok) {
      for (int g = flushed; g < ngroups && ok; ++g) ok = flush_group(g);
    }
    // every MMA is done once the last group was drained (or the CTA gave up): the ring is
    // idle and holds the z reduction
    float* zred = reinterpret_cast<float*>(ring);  // [kConvThreads][8]
    named_bar_sync(1, kConvThreads);
#pragma unroll
    for (int e = 0; e < 4; ++e) f32x2_split(zacc[e], zred[t * 8 + 2 * e], zred[t * 8 + 2 * e + 1]);
    named_bar_sync(1, kConvThreads);
    if (t < D) {
      const int uc = t / 8, e = t % 8;
      float zs = 0.f;
      for (int ph = 0; ph < kPhases; ++ph) zs += zred[(ph * kUnits + uc) * 8 + e];
      p.part_z[(static_cast<size_t>(bh) * p.nsplit + split) * D + t] = zs;
    }
    // S partial: S[k][n] for n = this lane's row and k in [col0, col0 + NC) (for each k the
    // warp's 32 lanes write 32 consecutive n: 128-byte stores)
    if (ok && drains) {
      float* dst = p.part_S + (static_cast<size_t>(bh) * p.nsplit + split) * D * D + n_row;
#pragma unroll
      for (int j = 0; j < NC; ++j) dst[static_cast<size_t>(col0 + j) * D] = acc[j];
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_d, C::kTmemCols);
  }
  // the grid completes only after the previous one (see the file comment)
  if (!p.wait_first) griddep_wait();
}

// S[bh] += sum_s part_S[bh][s], z[bh] += sum_s part_z[bh][s], slices in order; S_split[bh]
// (4 d^2 bytes a head) gets the new S as hi = bf16(S), lo = bf16(S - hi) in the tiles the
// hybrid attention's readout MMAs read: hi, then lo, each d/64 chunks of 64 columns n, a
// chunk d rows k of 128 bytes, 16-byte group g of row k at position g ^ (k % 8).
template <int D>
__global__ void __launch_bounds__(256) reduce_state_kernel(float* __restrict__ S, float* __restrict__ z,
                                                           uint8_t* __restrict__ S_split,
                                                           const float* __restrict__ part_S,
                                                           const float* __restrict__ part_z, int nsplit) {
  constexpr int kVec4PerHead = D * D / 4;
  constexpr int kCtasPerHead = (kVec4PerHead + 255) / 256;
  // the partials come from the previous grid; S and z may still be read by the one before
  griddep_wait();
  const int bh = blockIdx.x / kCtasPerHead;
  const int e4 = (blockIdx.x % kCtasPerHead) * 256 + threadIdx.x;
  if (e4 < kVec4PerHead) {
    float4* s4 = reinterpret_cast<float4*>(S + static_cast<size_t>(bh) * D * D) + e4;
    float4 acc = *s4;
    const float4* p4 = reinterpret_cast<const float4*>(part_S + static_cast<size_t>(bh) * nsplit * D * D) + e4;
    // all loads of a batch in flight (one L2 round trip for up to 16 slices), then the
    // adds in slice order
    constexpr int kBatch = 16;
    for (int s0 = 0; s0 < nsplit; s0 += kBatch) {
      float4 v[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u)
        if (s0 + u < nsplit) v[u] = __ldcg(p4 + static_cast<size_t>(s0 + u) * kVec4PerHead);
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        if (s0 + u < nsplit) {
          acc.x += v[u].x;
          acc.y += v[u].y;
          acc.z += v[u].z;
          acc.w += v[u].w;
        }
      }
    }
    *s4 = acc;
    // elements (k, n0 .. n0 + 3): half of a 16-byte group of the split tiles
    const int k = (4 * e4) / D, n0 = (4 * e4) % D;
    const uint32_t off = (n0 / 64) * (D * 128) + k * 128 + ((((n0 % 64) / 8) ^ (k & 7)) * 16) + (n0 % 8) * 2;
    const uint32_t h01 = pack_bf16x2(acc.x, acc.y), h23 = pack_bf16x2(acc.z, acc.w);
    const uint32_t l01 = pack_bf16x2(acc.x - bf16_lo_to_f32(h01), acc.y - bf16_hi_to_f32(h01));
    const uint32_t l23 = pack_bf16x2(acc.z - bf16_lo_to_f32(h23), acc.w - bf16_hi_to_f32(h23));
    uint8_t* sp = S_split + static_cast<size_t>(bh) * 4 * D * D + off;
    *reinterpret_cast<uint2*>(sp) = make_uint2(h01, h23);
    *reinterpret_cast<uint2*>(sp + 2 * D * D) = make_uint2(l01, l23);
  }
  if (blockIdx.x % kCtasPerHead == 0 && threadIdx.x < D) {
    float acc = z[static_cast<size_t>(bh) * D + threadIdx.x];
    for (int s = 0; s < nsplit; ++s) acc += __ldcg(part_z + (static_cast<size_t>(bh) * nsplit + s) * D + threadIdx.x);
    z[static_cast<size_t>(bh) * D + threadIdx.x] = acc;
  }
}

}  // namespace hf

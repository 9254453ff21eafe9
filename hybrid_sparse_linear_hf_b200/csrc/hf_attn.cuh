// Hybrid attention forward (hf_hybrid_attn_fwd): block-sparse softmax attention over
// the kept key blocks of the window + linear readout of the compact state, summed.
//
// Source: "Long-Horizon Streaming Video Generation via Hybrid Attention with
// Decoupled Distillation", German technical summary, section 2 A (block-sparse SWA
// computing only the Top-K blocks; linear temporal attention over a compact KV
// state; "Kombination": the output is the sum of both); Portuguese technical summary,
// section 2 A.
//
// One CTA per (b, h, query block I); the 128-row query tile holds block I's rows (for
// block < 128 the remaining rows are computed but never stored). 192 threads:
//   warp 0      TMA producer: Q tile once, then K/V of each kept block J into a ring
//               of kStages stages (row coordinate J*block; rows past Nk are zero-filled).
//   warp 1      TMEM owner (512 columns) + single-thread tcgen05 MMA issuer.
//   warps 2..5  128 "row" threads, thread <-> query row <-> TMEM lane: prologue
//               (phi(q) split into bf16 hi/lo written to TMEM, the state S converted to
//               bf16 hi/lo in shared memory, denominator phi(q).z + 1e-6 in fp32),
//               online softmax per block, epilogue (sum of both terms, bf16, TMA store).
// TMEM columns: [0,128) S buffer 0 (phi hi/lo during the prologue), [128,256) S
// buffer 1, [256,256+d) O accumulator, [384,384+d) linear term.
// Pipeline per kept block j: S_{j+1} = Q K_{j+1}^T is issued before O += P_j V_j so the
// tensor core works on the next scores while the row threads run the softmax of j. P_j
// is written as bf16 over the columns of S_j and read by the MMA straight from TMEM.
// Softmax is online in the log2 domain with a lazily raised running max: O is rescaled
// only when the block maximum exceeds the running max by more than 8 (a factor 256),
// which keeps exp2 arguments <= 8 and is exact since numerator and denominator share it.
// The linear term runs first: D_lin = phi_hi S_hi + phi_hi S_lo + phi_lo S_hi (two-term
// bf16 splits of phi(q) and S, fp32 accumulation); its S_hi/S_lo operands occupy the
// first ring stages, which the producer fills only after those MMAs completed.
#pragma once

#include "hf_ptx.cuh"

namespace hf {

constexpr uint32_t kKernAttn = 3;
constexpr int kAttnThreads = 192;
constexpr int kSmemLimit = 232448;  // max dynamic shared memory per CTA on sm_100

template <int D, int BLK>
struct AttnCfg {
  static constexpr int kChunks = D / 64;
  static constexpr int kQBytes = 128 * D * 2;
  static constexpr int kKVTileBytes = BLK * D * 2;
  static constexpr int kStageBytes = 2 * kKVTileBytes;
  static constexpr int kReadoutBytes = 2 * D * D * 2;  // S_hi + S_lo (bf16, d x d each)
  static constexpr int kStagesFit = (kSmemLimit - 2048 - 1024 - kQBytes) / kStageBytes;
  static constexpr int kStages = kStagesFit < 4 ? kStagesFit : 4;
  static constexpr int kReadoutStages = (kReadoutBytes + kStageBytes - 1) / kStageBytes;
  static_assert(kStages >= 2, "ring too small");
  static_assert(kReadoutStages <= kStages, "readout operands must fit in the ring");
  static constexpr int kDynSmem = 1024 + kQBytes + kStages * kStageBytes;
  static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256, kColLin = 384;
};

struct AttnParams {
  const int32_t* idx;  // [BH][nQB][r]
  const float* S;      // [BH][D][D]
  const float* z;      // [BH][D]
  int nQB, nKB, r;
  int last_len;        // valid tokens of key block nKB - 1
  float scale_log2;    // softmax scale * log2(e)
  unsigned long long timeout_ns;
  int inject;          // test only: the first S-ready commit is skipped
};

template <int D, int BLK>
__global__ void __launch_bounds__(kAttnThreads, 1)
    hybrid_attn_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
                       const __grid_constant__ CUtensorMap mapV, const __grid_constant__ CUtensorMap mapO,
                       AttnParams p) {
  using C = AttnCfg<D, BLK>;
  constexpr int NS = C::kStages;
  constexpr int KR = C::kReadoutStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                  // Q tile; reused as the output staging tile
  uint8_t* ring = smem + C::kQBytes;   // NS stages of [K tile | V tile]; S_hi/S_lo first

  __shared__ uint64_t q_bar, full_bar[NS], empty_bar[NS];
  __shared__ uint64_t pro_bar, sfull_bar[2], pfull_bar[2], odone_bar, lin_bar, final_bar, drain_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int bh = blockIdx.x / p.nQB;
  const int I = blockIdx.x % p.nQB;
  const int32_t* idx_row = p.idx + (static_cast<size_t>(bh) * p.nQB + I) * p.r;
  volatile int* abort_flag = &abort_sh;

  if (threadIdx.x == 0) {
    mbar_init(&q_bar, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(&pro_bar, 128);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sfull_bar[b], 1);
      mbar_init(&pfull_bar[b], 128);
    }
    mbar_init(&odone_bar, 1);
    mbar_init(&lin_bar, 1);
    mbar_init(&final_bar, 1);
    mbar_init(&drain_bar, 1);
    abort_sh = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&mapQ);
    tma_prefetch_desc(&mapK);
    tma_prefetch_desc(&mapV);
    tma_prefetch_desc(&mapO);
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  if (warp == 0) {
    // ============================ TMA producer ============================
    if (lane == 0) {
      mbar_arrive_expect_tx(&q_bar, C::kQBytes);
#pragma unroll
      for (int c = 0; c < C::kChunks; ++c) tma_load_3d(sQ + c * 128 * 128, &mapQ, &q_bar, c * 64, I * BLK, bh);
      int v = KR;  // virtual block index: the readout used virtual blocks [0, KR)
      bool bad = false;
      for (int jj = 0; jj < p.r; ++jj) {
        const int J = __ldg(idx_row + jj);
        if (J < 0 || J >= p.nKB) {
          bad = true;
          continue;
        }
        const int s = v % NS, u = v / NS;
        if (u >= 1 && !mbar_wait(&empty_bar[s], (u - 1) & 1, abort_flag, p.timeout_ns, (kKernAttn << 8) | 1))
          break;
        if (*abort_flag) break;
        uint8_t* st = ring + s * C::kStageBytes;
        mbar_arrive_expect_tx(&full_bar[s], C::kStageBytes);
#pragma unroll
        for (int c = 0; c < C::kChunks; ++c) {
          tma_load_3d(st + c * BLK * 128, &mapK, &full_bar[s], c * 64, J * BLK, bh);
          tma_load_3d(st + C::kKVTileBytes + c * BLK * 128, &mapV, &full_bar[s], c * 64, J * BLK, bh);
        }
        ++v;
      }
      if (bad) atomicCAS(&g_hf_error_word, 0u, (0x7200u << 16) | (kKernAttn << 8));
      // drain: the last NS fills (and the Q tile) must have landed before exit
      mbar_wait_drain(&q_bar, 0, p.timeout_ns, (kKernAttn << 8) | 2);
      for (int vv = max(KR, v - NS); vv < v; ++vv) {
        const int s = vv % NS, u = vv / NS;
        mbar_wait_drain(&full_bar[s], (u - (s < KR ? 1 : 0)) & 1, p.timeout_ns, (kKernAttn << 8) | 3);
      }
    }
  } else if (warp == 1) {
    // ============================ MMA issuer ============================
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, BLK, false, false);  // A=Q, B=K: both K-major
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, false, true);     // A=P (TMEM), B=V: MN-major
      constexpr uint32_t idesc_lin = idesc_bf16_f32(128, D, false, true);    // A=phi (TMEM), B=S: MN-major
      int n = 0;
      for (int jj = 0; jj < p.r; ++jj) {
        const int J = __ldg(idx_row + jj);
        n += (J >= 0 && J < p.nKB);
      }
      const uint32_t q_addr = smem_u32(sQ);
      const uint32_t ring_addr = smem_u32(ring);
      bool ok = mbar_wait(&q_bar, 0, abort_flag, p.timeout_ns, (kKernAttn << 8) | 4) &&
                mbar_wait(&pro_bar, 0, abort_flag, p.timeout_ns, (kKernAttn << 8) | 5);
      if (ok) {
        tc_fence_after();
        // linear term: D_lin = phi_hi S_hi + phi_hi S_lo + phi_lo S_hi
        const uint32_t s_hi = ring_addr, s_lo = ring_addr + D * D * 2;
        int step = 0;
#pragma unroll
        for (int term = 0; term < 3; ++term) {
          const uint32_t a_col = (term == 2) ? D / 2 : 0;
          const uint32_t b_base = (term == 1) ? s_lo : s_hi;
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks, ++step) {
            const uint64_t bdesc = sdesc_sw128(b_base + ks * 2048, D * 128, 1024);
            umma_ts(tmem + C::kColLin, tmem + C::kColS0 + a_col + ks * 8, bdesc, idesc_lin, step > 0 ? 1u : 0u);
          }
        }
#pragma unroll
        for (int s = 0; s < KR; ++s) umma_commit(&empty_bar[s]);
        umma_commit(&lin_bar);
      }
      auto stage_of = [&](int j, int& s, uint32_t& par) {
        const int vv = j + KR;
        s = vv % NS;
        par = static_cast<uint32_t>((vv / NS) - (s < KR ? 1 : 0)) & 1u;
      };
      auto issue_qk = [&](int j) {
        int s;
        uint32_t par;
        stage_of(j, s, par);
        if (!mbar_wait(&full_bar[s], par, abort_flag, p.timeout_ns, (kKernAttn << 8) | 6)) return false;
        tc_fence_after();
        const uint32_t k_addr = ring_addr + s * C::kStageBytes;
        const uint32_t d_col = (j & 1) ? C::kColS1 : C::kColS0;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t koff = (ks / 4) * (128 * 128) + (ks % 4) * 32;
          const uint32_t boff = (ks / 4) * (BLK * 128) + (ks % 4) * 32;
          umma_ss(tmem + d_col, sdesc_sw128(q_addr + koff, 16, 1024), sdesc_sw128(k_addr + boff, 16, 1024),
                  idesc_qk, ks > 0 ? 1u : 0u);
        }
        if (!(p.inject && j == 0)) umma_commit(&sfull_bar[j & 1]);
        return true;
      };
      if (ok && n > 0) ok = issue_qk(0);
      for (int j = 0; j < n && ok; ++j) {
        if (j + 1 < n && !(ok = issue_qk(j + 1))) break;
        if (!(ok = mbar_wait(&pfull_bar[j & 1], (j >> 1) & 1, abort_flag, p.timeout_ns, (kKernAttn << 8) | 7)))
          break;
        tc_fence_after();
        int s;
        uint32_t par;
        stage_of(j, s, par);
        const uint32_t v_addr = ring_addr + s * C::kStageBytes + C::kKVTileBytes;
        const uint32_t p_col = (j & 1) ? C::kColS1 : C::kColS0;
#pragma unroll
        for (int ks = 0; ks < BLK / 16; ++ks) {
          umma_ts(tmem + C::kColO, tmem + p_col + ks * 8, sdesc_sw128(v_addr + ks * 2048, BLK * 128, 1024),
                  idesc_pv, (j > 0 || ks > 0) ? 1u : 0u);
        }
        umma_commit(&empty_bar[s]);
        umma_commit(&odone_bar);
      }
      if (ok) umma_commit(&final_bar);
      umma_commit(&drain_bar);
      mbar_wait_drain(&drain_bar, 0, p.timeout_ns, (kKernAttn << 8) | 8);
    }
  } else {
    // ======================= row threads (softmax, epilogue) =======================
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;  // query row within the tile == TMEM lane
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    // tcgen05.ld/st are warp-collective: every wait that guards one is made warp-uniform
    bool ok = __all_sync(0xffffffffu, mbar_wait(&q_bar, 0, abort_flag, p.timeout_ns, (kKernAttn << 8) | 9));
    float den = 1.0f;
    if (ok) {
      // ---- prologue: phi(q) hi/lo -> TMEM, den = phi(q).z + 1e-6, S -> bf16 hi/lo in smem
      const float* zrow = p.z + static_cast<size_t>(bh) * D;
      float dacc = 0.f;
#pragma unroll
      for (int g = 0; g < D / 32; ++g) {  // 32 elements -> 16 packed columns of hi and of lo
        uint32_t hi[16], lo[16];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const int unit = g * 4 + h;  // 16-byte unit of the row: elements [8*unit, 8*unit + 8)
          const uint32_t off = (unit / 8) * (128 * 128) + row * 128 + (((unit % 8) ^ (row & 7)) * 16);
          const uint4 qv = *reinterpret_cast<const uint4*>(sQ + off);
          const uint32_t w[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float x0 = bf16_lo_to_f32(w[e]), x1 = bf16_hi_to_f32(w[e]);
            const float p0 = x0 > 0.f ? x0 + 1.f : __expf(x0);
            const float p1 = x1 > 0.f ? x1 + 1.f : __expf(x1);
            const float2 zz = __ldg(reinterpret_cast<const float2*>(zrow + unit * 8 + 2 * e));
            dacc = fmaf(p0, zz.x, dacc);
            dacc = fmaf(p1, zz.y, dacc);
            const uint32_t hh = pack_bf16x2(p0, p1);
            hi[h * 4 + e] = hh;
            lo[h * 4 + e] = pack_bf16x2(p0 - bf16_lo_to_f32(hh), p1 - bf16_hi_to_f32(hh));
          }
        }
        // TMEM column c holds elements (2c, 2c+1) of the row: hi at [0, D/2), lo at [D/2, D)
        tmem_st16(lane_addr + C::kColS0 + g * 16, hi);
        tmem_st16(lane_addr + C::kColS0 + D / 2 + g * 16, lo);
      }
      den = dacc + 1e-6f;
      // state rows: thread k < D converts S[bh][k][:] into MN-major bf16 hi/lo tiles
      if (row < D) {
        const float* srow = p.S + (static_cast<size_t>(bh) * D + row) * D;
        uint8_t* s_hi = ring;
        uint8_t* s_lo = ring + D * D * 2;
#pragma unroll 4
        for (int unit = 0; unit < D / 8; ++unit) {
          const float4 a = __ldg(reinterpret_cast<const float4*>(srow + unit * 8));
          const float4 b = __ldg(reinterpret_cast<const float4*>(srow + unit * 8 + 4));
          const float f[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
          uint32_t hv[4], lv[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const uint32_t hh = pack_bf16x2(f[2 * e], f[2 * e + 1]);
            hv[e] = hh;
            lv[e] = pack_bf16x2(f[2 * e] - bf16_lo_to_f32(hh), f[2 * e + 1] - bf16_hi_to_f32(hh));
          }
          const uint32_t off = (unit / 8) * (D * 128) + row * 128 + (((unit % 8) ^ (row & 7)) * 16);
          *reinterpret_cast<uint4*>(s_hi + off) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
          *reinterpret_cast<uint4*>(s_lo + off) = make_uint4(lv[0], lv[1], lv[2], lv[3]);
        }
      }
      fence_proxy_async_smem();
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&pro_bar);
    }

    // ---- online softmax over the kept blocks
    float m_run = -INFINITY, l_run = 0.f;
    int j = 0;
    for (int jj = 0; jj < p.r && ok; ++jj) {
      const int J = __ldg(idx_row + jj);
      if (J < 0 || J >= p.nKB) continue;
      const int b = j & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&sfull_bar[b], (j >> 1) & 1, abort_flag, p.timeout_ns,
                                             (kKernAttn << 8) | 10));
      if (!ok) break;
      tc_fence_after();
      const uint32_t s_addr = lane_addr + (b ? C::kColS1 : C::kColS0);
      uint32_t sr[BLK];
#pragma unroll
      for (int c = 0; c < BLK; c += 32) tmem_ld32(s_addr + c, sr + c);
      tmem_wait_ld();
      reg_fence<BLK>(sr);
      float* s = reinterpret_cast<float*>(sr);
      const int valid = (J == p.nKB - 1) ? p.last_len : BLK;
      if (valid < BLK) {
#pragma unroll
        for (int c = 0; c < BLK; ++c)
          if (c >= valid) s[c] = -INFINITY;
      }
      float mx = s[0];
#pragma unroll
      for (int c = 1; c < BLK; ++c) mx = fmaxf(mx, s[c]);
      mx *= p.scale_log2;
      if (j == 0) {
        m_run = mx;
      } else {
        // A row raises its running max only when the block max exceeds it by more than
        // 8 (log2 units); the O rescale is done by the whole warp whenever any of its
        // rows needs it (alpha = 1 for the others), since TMEM access is warp-collective.
        const bool need = mx > m_run + 8.0f;
        if (__any_sync(0xffffffffu, need)) {
          const float alpha = need ? ex2_approx(m_run - mx) : 1.0f;
          ok = __all_sync(0xffffffffu, mbar_wait(&odone_bar, (j - 1) & 1, abort_flag, p.timeout_ns,
                                                 (kKernAttn << 8) | 11));
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < D; c += 32) {
            uint32_t o[32];
            tmem_ld32(lane_addr + C::kColO + c, o);
            tmem_wait_ld();
            reg_fence<32>(o);
#pragma unroll
            for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
            tmem_st32(lane_addr + C::kColO + c, o);
          }
          if (need) {
            l_run *= alpha;
            m_run = mx;
          }
        }
      }
      float lsum = 0.f;
      uint32_t pk[BLK / 2];
#pragma unroll
      for (int c = 0; c < BLK; c += 2) {
        const float p0 = ex2_approx(fmaf(s[c], p.scale_log2, -m_run));
        const float p1 = ex2_approx(fmaf(s[c + 1], p.scale_log2, -m_run));
        lsum += p0 + p1;
        pk[c / 2] = pack_bf16x2(p0, p1);
      }
      l_run += lsum;
#pragma unroll
      for (int c = 0; c < BLK / 2; c += 16) tmem_st16(s_addr + c, pk + c);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&pfull_bar[b]);
      ++j;
    }

    // ---- epilogue: O = O_s / l + O_lin / den -> bf16 -> TMA store of the block's rows
    if (ok) ok = mbar_wait(&final_bar, 0, abort_flag, p.timeout_ns, (kKernAttn << 8) | 12) &&
                 mbar_wait(&lin_bar, 0, abort_flag, p.timeout_ns, (kKernAttn << 8) | 13);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      tc_fence_after();
      const float inv_l = (j > 0 && l_run > 0.f) ? 1.0f / l_run : 0.0f;
      const float inv_den = 1.0f / den;
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        uint32_t o[32], lin[32];
        tmem_ld32(lane_addr + C::kColO + c, o);
        tmem_ld32(lane_addr + C::kColLin + c, lin);
        tmem_wait_ld();
        reg_fence<32>(o);
        reg_fence<32>(lin);
        if (row < BLK) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {  // four 16-byte units of 8 columns
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int k = u * 8 + 2 * e;
              const float y0 = (j > 0 ? __uint_as_float(o[k]) * inv_l : 0.f) + __uint_as_float(lin[k]) * inv_den;
              const float y1 =
                  (j > 0 ? __uint_as_float(o[k + 1]) * inv_l : 0.f) + __uint_as_float(lin[k + 1]) * inv_den;
              w[e] = pack_bf16x2(y0, y1);
            }
            const int unit = c / 8 + u;
            const uint32_t off = (unit / 8) * (BLK * 128) + row * 128 + (((unit % 8) ^ (row & 7)) * 16);
            *reinterpret_cast<uint4*>(sQ + off) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
      fence_proxy_async_smem();
    }
    named_bar_sync(1, 128);
    if (ok && threadIdx.x == 64) {
#pragma unroll
      for (int c = 0; c < C::kChunks; ++c) tma_store_3d(&mapO, sQ + c * BLK * 128, c * 64, I * BLK, bh);
      tma_store_commit();
      tma_store_wait_all();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace hf

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
// block < 128 the remaining rows are computed but never stored). 384 threads, three
// warpgroups; setmaxnreg moves registers from the first to the other two:
//   warp 0      TMA producer of the Q tile (once) and of the K tile of each kept block J
//               into a ring of K slots (row coordinate J*block; rows past Nk are
//               zero-filled); a K slot frees as soon as its QK^T is done.
//   warp 1      TMEM owner (512 columns) + single-thread tcgen05 MMA issuer.
//   warp 2      TMA producer of the V tiles into a ring of V slots. (warp 3 idles)
//   warps 4..11 row threads: warps w and w+4 share TMEM lane quarter w % 4 (query rows
//               32*(w%4) .. +31); warps 4..7 exponentiate the first half of every row's
//               columns, warps 8..11 the second half: two softmax warps per sub-partition.
// TMEM columns: S buffers [0,128) and [128,256), O [256, 256+d), Q [384, 384+d/2)
// (bf16 pairs), P [448, 448+block/2) (bf16 pairs).
// Shared-memory traffic is the binding resource at d = block = 128 (one SMEM operand of
// 128x128x16 per 64 tensor cycles is already 128 B/clk): Q therefore lives in TMEM
// (S = Q K^T reads only K from shared memory) and P too (O += P V reads only V).
// Pipeline per kept block j: S_j -> buffer j%2; the row threads load S_j into registers
// and release the buffer at once, so S_{j+2} is computed during softmax j; P_j goes to
// the P region once PV_{j-1} has read P_{j-1}; PV_j follows P_j.
// Softmax: online in the log2 domain with a lazily raised running max (O is rescaled only
// when a block maximum exceeds the running max by more than 8, i.e. a factor 256; exact
// since numerator and denominator share the max); both warps of a quarter read the whole
// S row and take the same full-row max (no exchange, so they never wait on each other),
// each exponentiating its half; the O rescale is warp-uniform because TMEM access is
// warp-collective; 3 exp2 pairs in 8 run on the FMA pipe, the rest on MUFU.
// Linear term, after the last block: phi(q) in fp32 split into bf16 hi + lo (TMEM, S
// buffer 1), the state S split into bf16 hi + lo (shared memory, over the idle rings),
// D_lin = phi_hi S_hi + phi_hi S_lo + phi_lo S_hi on the tensor cores (TMEM, S buffer
// 0), denominator phi(q).z + 1e-6 in fp32; the epilogue writes O_s / l + D_lin / den.
#pragma once

#include <type_traits>

#include "hf_ptx.cuh"

namespace hf {

constexpr uint32_t kKernAttn = 3;
constexpr int kAttnThreads = 384;
constexpr int kRegsSupport = 104;   // registers per thread, producer/MMA warpgroup
constexpr int kRegsRows = 200;     // registers per thread, row warpgroups
static_assert(128 * kRegsSupport + 256 * kRegsRows <= kAttnThreads * 168, "setmaxnreg split exceeds the launch");
constexpr int kSmemLimit = 232448;  // max dynamic shared memory per CTA on sm_100
constexpr int kPolyOf8 = 3;         // pairs (of every 8) that take exp2 on the FMA pipe

template <int D, int BLK>
struct AttnCfg {
  static constexpr int kChunks = D / 64;
  static constexpr int kQBytes = 128 * D * 2;
  static constexpr int kKVTileBytes = BLK * D * 2;
  static constexpr int kReadoutBytes = 2 * D * D * 2;  // S_hi + S_lo (bf16, d x d each)
  // K slots free right after their QK^T, V slots only after their PV, two softmax periods
  // before the slot is needed again: K gets the deeper ring.
  static constexpr int kTiles = (kSmemLimit - 6144 - 1024 - kQBytes) / kKVTileBytes;
  static constexpr int kKSlots = ((kTiles + 1) / 2) < 4 ? ((kTiles + 1) / 2) : 4;
  static constexpr int kVSlots = (kTiles - kKSlots) < 4 ? (kTiles - kKSlots) : 4;
  static_assert(kKSlots >= 2 && kVSlots >= 2, "ring too small");
  static_assert(kReadoutBytes <= (kKSlots + kVSlots) * kKVTileBytes, "readout operands must fit in the rings");
  static constexpr int kDynSmem = 1024 + kQBytes + (kKSlots + kVSlots) * kKVTileBytes;
  static constexpr uint32_t kColS = 0;      // S buffers at 0 and 128
  static constexpr uint32_t kColO = 256;
  static constexpr uint32_t kColQ = 384;
  static constexpr uint32_t kColP = 448;
  static constexpr uint32_t kColLin = 0;    // linear term (after the last block)
  static constexpr uint32_t kColPhi = 128;  // phi(q) hi | lo (after the last block)
  static constexpr int kHB = BLK / 2;       // S columns per half-row thread
  static constexpr int kHD = D / 2;         // O columns per half-row thread
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
  constexpr int NSK = C::kKSlots;
  constexpr int NSV = C::kVSlots;
  constexpr int HB = C::kHB;
  constexpr int HD = C::kHD;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                             // Q tile; reused as the output staging tile
  uint8_t* kring = smem + C::kQBytes;              // NSK K slots
  uint8_t* vring = kring + NSK * C::kKVTileBytes;  // NSV V slots (S_hi/S_lo over both rings at the end)

  __shared__ uint64_t q_bar, qt_bar, kfull_bar[NSK], kempty_bar[NSK], vfull_bar[NSV], vempty_bar[NSV];
  __shared__ uint64_t sfull_bar[2], sfree_bar[2], pfull_bar, pdone_bar[2], xch_bar[4];
  __shared__ uint64_t final_bar, pro_bar, lin_bar, drain_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  __shared__ float z_sh[D];
  __shared__ float xend[2][2][128];  // end-of-tile exchange: [den | l][half][row]

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int bh = blockIdx.x / p.nQB;
  const int I = blockIdx.x % p.nQB;
  const int32_t* idx_row = p.idx + (static_cast<size_t>(bh) * p.nQB + I) * p.r;
  volatile int* abort_flag = &abort_sh;

  if (threadIdx.x == 0) {
    mbar_init(&q_bar, 1);
    mbar_init(&qt_bar, 256);
    for (int s = 0; s < NSK; ++s) {
      mbar_init(&kfull_bar[s], 1);
      mbar_init(&kempty_bar[s], 1);
    }
    for (int s = 0; s < NSV; ++s) {
      mbar_init(&vfull_bar[s], 1);
      mbar_init(&vempty_bar[s], 1);
    }
    for (int q = 0; q < 4; ++q) mbar_init(&xch_bar[q], 64);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sfull_bar[b], 1);
      mbar_init(&sfree_bar[b], 256);
      mbar_init(&pdone_bar[b], 1);
    }
    mbar_init(&pfull_bar, 256);
    mbar_init(&final_bar, 1);
    mbar_init(&pro_bar, 256);
    mbar_init(&lin_bar, 1);
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
  for (int i = threadIdx.x; i < D; i += kAttnThreads) z_sh[i] = p.z[static_cast<size_t>(bh) * D + i];
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  if (warp < 4) {
   // warpgroup 0: producers and MMA issuer give registers to the row warpgroups
   warpgroup_reg_dec<kRegsSupport>();
   if (warp == 0 || warp == 2) {
    // ============================ TMA producers ============================
    if (lane == 0) {
      const bool is_k = warp == 0;  // warp 0: Q + K tiles, warp 2: V tiles
      const CUtensorMap* map = is_k ? &mapK : &mapV;
      uint64_t* full = is_k ? kfull_bar : vfull_bar;
      uint64_t* empty = is_k ? kempty_bar : vempty_bar;
      uint8_t* slots = is_k ? kring : vring;
      const int NS = is_k ? NSK : NSV;
      if (is_k) {
        mbar_arrive_expect_tx(&q_bar, C::kQBytes);
#pragma unroll
        for (int c = 0; c < C::kChunks; ++c) tma_load_3d(sQ + c * 128 * 128, &mapQ, &q_bar, c * 64, I * BLK, bh);
      }
      int v = 0;  // kept-block counter (valid indices only)
      bool bad = false;
      for (int jj = 0; jj < p.r; ++jj) {
        const int J = __ldg(idx_row + jj);
        if (J < 0 || J >= p.nKB) {
          bad = true;
          continue;
        }
        const int s = v % NS, u = v / NS;
        if (u >= 1 && !mbar_wait(&empty[s], (u - 1) & 1, abort_flag, p.timeout_ns, (kKernAttn << 8) | 1)) break;
        if (*abort_flag) break;
        uint8_t* dst = slots + s * C::kKVTileBytes;
        mbar_arrive_expect_tx(&full[s], C::kKVTileBytes);
#pragma unroll
        for (int c = 0; c < C::kChunks; ++c) tma_load_3d(dst + c * BLK * 128, map, &full[s], c * 64, J * BLK, bh);
        ++v;
      }
      if (bad && is_k) atomicCAS(&g_hf_error_word, 0u, (0x7200u << 16) | (kKernAttn << 8));
      // drain: the Q tile and the last NS fills must have landed before exit
      if (is_k) mbar_wait_drain(&q_bar, 0, p.timeout_ns, (kKernAttn << 8) | 2);
      for (int vv = max(0, v - NS); vv < v; ++vv)
        mbar_wait_drain(&full[vv % NS], (vv / NS) & 1, p.timeout_ns, (kKernAttn << 8) | 3);
    }
   } else if (warp == 1) {
    // ============================ MMA issuer ============================
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, BLK, false, false);  // A=Q (TMEM), B=K: K-major
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, false, true);     // A=P (TMEM), B=V: MN-major
      constexpr uint32_t idesc_lin = idesc_bf16_f32(128, D, false, true);    // A=phi (TMEM), B=S: MN-major
      int n = 0;
      for (int jj = 0; jj < p.r; ++jj) {
        const int J = __ldg(idx_row + jj);
        n += (J >= 0 && J < p.nKB);
      }
      // Descriptors are built once; an MMA only adds a constant offset (in 16-byte units)
      // to the 14-bit start-address field (shared-memory addresses stay below 256 KB, so the
      // field never carries). This keeps the single issuing thread ahead of the tensor core.
      const uint64_t kdesc = sdesc_sw128(smem_u32(kring), 16, 1024);
      const uint64_t vdesc = sdesc_sw128(smem_u32(vring), BLK * 128, 1024);
      auto issue_qk = [&](int j) {
        const int s = j % NSK;
        if (!mbar_wait(&kfull_bar[s], (j / NSK) & 1, abort_flag, p.timeout_ns, (kKernAttn << 8) | 6)) return false;
        tc_fence_after();
        const uint64_t kd = kdesc + static_cast<uint64_t>((s * C::kKVTileBytes) >> 4);
        const uint32_t d_tmem = tmem + C::kColS + (j & 1) * 128;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          constexpr int kKChunk = (BLK * 128) >> 4;
          umma_ts(d_tmem, tmem + C::kColQ + ks * 8, kd + (ks / 4) * kKChunk + (ks % 4) * 2, idesc_qk,
                  ks > 0 ? 1u : 0u);
        }
        umma_commit(&kempty_bar[s]);
        if (!(p.inject && j == 0)) umma_commit(&sfull_bar[j & 1]);
        return true;
      };
      bool ok = mbar_wait(&qt_bar, 0, abort_flag, p.timeout_ns, (kKernAttn << 8) | 4);
      for (int j = 0; j < 2 && j < n && ok; ++j) ok = issue_qk(j);
      for (int j = 0; j < n && ok; ++j) {
        // S_{j+2} into buffer j%2 as soon as the row threads hold S_j in registers
        if (j + 2 < n) {
          ok = mbar_wait(&sfree_bar[j & 1], (j >> 1) & 1, abort_flag, p.timeout_ns, (kKernAttn << 8) | 15) &&
               issue_qk(j + 2);
          if (!ok) break;
        }
        const int s = j % NSV;
        if (!(ok = mbar_wait(&pfull_bar, j & 1, abort_flag, p.timeout_ns, (kKernAttn << 8) | 7) &&
                   mbar_wait(&vfull_bar[s], (j / NSV) & 1, abort_flag, p.timeout_ns, (kKernAttn << 8) | 14)))
          break;
        tc_fence_after();
        const uint64_t vd = vdesc + static_cast<uint64_t>((s * C::kKVTileBytes) >> 4);
#pragma unroll
        for (int ks = 0; ks < BLK / 16; ++ks)
          umma_ts(tmem + C::kColO, tmem + C::kColP + ks * 8, vd + ks * 128, idesc_pv, (j > 0 || ks > 0) ? 1u : 0u);
        umma_commit(&vempty_bar[s]);
        umma_commit(&pdone_bar[j & 1]);
      }
      if (ok) {
        umma_commit(&final_bar);
        // linear term: D_lin = phi_hi S_hi + phi_hi S_lo + phi_lo S_hi
        if ((ok = mbar_wait(&pro_bar, 0, abort_flag, p.timeout_ns, (kKernAttn << 8) | 5))) {
          tc_fence_after();
          const uint64_t sdesc_hi = sdesc_sw128(smem_u32(kring), D * 128, 1024);
          const uint64_t sdesc_lo = sdesc_hi + ((D * D * 2) >> 4);
#pragma unroll
          for (int term = 0; term < 3; ++term) {
            const uint32_t a_col = C::kColPhi + ((term == 2) ? D / 2 : 0);
            const uint64_t b = (term == 1) ? sdesc_lo : sdesc_hi;
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks)
              umma_ts(tmem + C::kColLin, tmem + a_col + ks * 8, b + ks * 128, idesc_lin,
                      (term > 0 || ks > 0) ? 1u : 0u);
          }
          umma_commit(&lin_bar);
        }
      }
      umma_commit(&drain_bar);
      mbar_wait_drain(&drain_bar, 0, p.timeout_ns, (kKernAttn << 8) | 8);
    }
   }
  } else {
    warpgroup_reg_inc<kRegsRows>();
    // ======================= row threads (softmax, readout, epilogue) =======================
    const int quarter = warp & 3;
    const int half = (warp - 4) >> 2;     // 0: warps 4..7, 1: warps 8..11
    const int row = quarter * 32 + lane;  // query row within the tile == TMEM lane
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    // the two warps of a lane quarter meet once, at the end, on xch_bar[quarter]
    // (an mbarrier: bounded wait)
    uint64_t* pair_bar = &xch_bar[quarter];
    // tcgen05.ld/st are warp-collective: every wait that guards one is made warp-uniform
    bool ok = __all_sync(0xffffffffu, mbar_wait(&q_bar, 0, abort_flag, p.timeout_ns, (kKernAttn << 8) | 9));
    if (ok) {
      // Q row -> TMEM as bf16 pairs (the A operand of S = Q K^T); this half's elements
#pragma unroll
      for (int g = 0; g < HD / 32; ++g) {
        uint32_t w[16];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const int unit = half * (HD / 8) + g * 4 + h;
          const uint32_t off = (unit / 8) * (128 * 128) + row * 128 + (((unit % 8) ^ (row & 7)) * 16);
          const uint4 qv = *reinterpret_cast<const uint4*>(sQ + off);
          w[h * 4 + 0] = qv.x;
          w[h * 4 + 1] = qv.y;
          w[h * 4 + 2] = qv.z;
          w[h * 4 + 3] = qv.w;
        }
        tmem_st16(lane_addr + C::kColQ + half * (HD / 2) + g * 16, w);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&qt_bar);
    }

    // ---- online softmax over the kept blocks (this thread: columns [half*HB, half*HB+HB))
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
      // the whole row of S_j: the full-row max is computed by both warps of the quarter
      // (no exchange between them); each keeps only its half for the exponentials
      uint32_t sr[BLK];
      tmem_ld_cols<BLK>(lane_addr + C::kColS + b * 128, sr);
      tmem_wait_ld();
      reg_fence<BLK>(sr);
      tc_fence_before();
      mbar_arrive(&sfree_bar[b]);  // S_j is in registers: the buffer may take S_{j+2}
      float* srow = reinterpret_cast<float*>(sr);
      const int valid = (J == p.nKB - 1) ? p.last_len : BLK;
      if (valid < BLK) {  // partial last key block: padding columns are masked out
#pragma unroll
        for (int c = 0; c < BLK; ++c)
          if (c >= valid) srow[c] = -INFINITY;
      }
      // row max: 8 independent chains of 3-input max
      float mc[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mc[k] = fmaxf(srow[k], srow[k + 8]);
#pragma unroll
      for (int c = 16; c < BLK; c += 16) {
#pragma unroll
        for (int k = 0; k < 8; ++k) mc[k] = fmax3(mc[k], srow[c + k], srow[c + 8 + k]);
      }
      const float mx =
          fmax3(fmax3(mc[0], mc[1], mc[2]), fmax3(mc[3], mc[4], mc[5]), fmaxf(mc[6], mc[7])) * p.scale_log2;
      bool o_ready = j == 0;  // PV_{j-1} done (O final for j-1, P region free)
      if (j == 0) {
        m_run = mx;
      } else {
        // A row raises its running max only when the block max exceeds it by more than
        // 8 (log2 units); the O rescale is done by the whole warp whenever any of its
        // rows needs it (alpha = 1 for the others); it waits for PV_{j-1}.
        const bool need = mx > m_run + 8.0f;
        if (__any_sync(0xffffffffu, need)) {
          const float alpha = need ? ex2_approx(m_run - mx) : 1.0f;
          ok = __all_sync(0xffffffffu, mbar_wait(&pdone_bar[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag,
                                                 p.timeout_ns, (kKernAttn << 8) | 11));
          if (!ok) break;
          o_ready = true;
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < HD; c += 32) {
            uint32_t o[32];
            tmem_ld32(lane_addr + C::kColO + half * HD + c, o);
            tmem_wait_ld();
            reg_fence<32>(o);
#pragma unroll
            for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
            tmem_st32(lane_addr + C::kColO + half * HD + c, o);
          }
          if (need) {
            l_run *= alpha;
            m_run = mx;
          }
        }
      }
      // p = 2^(s * scale * log2 e - m) over this warp's half of the row: packed fp32 pairs;
      // kPolyOf8 pairs of every 8 run exp2 on the FMA pipe, the others on MUFU, so neither
      // unit alone sets the pace. The half is a compile-time offset (a runtime index into
      // the register array would move it to local memory).
      uint32_t pk[HB / 2];
      auto exp_half = [&](auto off) {
        constexpr int OFF = decltype(off)::value;
        const uint64_t sl2 = f32x2(p.scale_log2, p.scale_log2);
        const uint64_t nm2 = f32x2(-m_run, -m_run);
        uint64_t lacc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int c = 0; c < HB; c += 2) {
          const uint64_t x2 = ffma2(f32x2(srow[OFF + c], srow[OFF + c + 1]), sl2, nm2);
          float p0, p1;
          if (((c / 2) & 7) >= 8 - kPolyOf8) {
            exp2_poly_x2(x2, p0, p1);
          } else {
            float x0, x1;
            f32x2_split(x2, x0, x1);
            p0 = ex2_approx(x0);
            p1 = ex2_approx(x1);
          }
          lacc[(c / 2) & 3] = fadd2(lacc[(c / 2) & 3], f32x2(p0, p1));
          pk[c / 2] = pack_bf16x2(p0, p1);
        }
        const uint64_t l2 = fadd2(fadd2(lacc[0], lacc[1]), fadd2(lacc[2], lacc[3]));
        float la, lb;
        f32x2_split(l2, la, lb);
        l_run += la + lb;
      };
      // p = 2^(s * scale * log2 e - m) over this warp's half of the row: packed fp32 pairs;
      // kPolyOf8 pairs of every 8 run exp2 on the FMA pipe, the others on MUFU, so neither
      // unit alone sets the pace. The half is a compile-time offset (a runtime index into
      // the register array would move it to local memory).
      if (half == 0) {
        exp_half(std::integral_constant<int, 0>{});
      } else {
        exp_half(std::integral_constant<int, HB>{});
      }
      // P_j -> the P region once PV_{j-1} has read P_{j-1} (normally long done by now)
      if (!o_ready) {
        ok = __all_sync(0xffffffffu, mbar_wait(&pdone_bar[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag,
                                               p.timeout_ns, (kKernAttn << 8) | 16));
        if (!ok) break;
        tc_fence_after();
      }
      tmem_st_cols<HB / 2>(lane_addr + C::kColP + half * (HB / 2), pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&pfull_bar);
      ++j;
    }

    // ---- linear term operands (all PV done: the S buffers and both rings are free)
    ok = ok && mbar_wait(&final_bar, 0, abort_flag, p.timeout_ns, (kKernAttn << 8) | 12);
    ok = __all_sync(0xffffffffu, ok);
    float den = 1.0f, l_tot = 0.f;
    if (ok) {
      tc_fence_after();
      float dacc = 0.f;
#pragma unroll
      for (int g = 0; g < HD / 32; ++g) {  // 32 elements -> 16 packed columns of hi and of lo
        uint32_t hi[16], lo[16];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const int unit = half * (HD / 8) + g * 4 + h;  // elements [8*unit, 8*unit + 8)
          const uint32_t off = (unit / 8) * (128 * 128) + row * 128 + (((unit % 8) ^ (row & 7)) * 16);
          const uint4 qv = *reinterpret_cast<const uint4*>(sQ + off);
          const uint32_t w[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float x0 = bf16_lo_to_f32(w[e]), x1 = bf16_hi_to_f32(w[e]);
            const float p0 = x0 > 0.f ? x0 + 1.f : __expf(x0);
            const float p1 = x1 > 0.f ? x1 + 1.f : __expf(x1);
            dacc = fmaf(p0, z_sh[unit * 8 + 2 * e], dacc);
            dacc = fmaf(p1, z_sh[unit * 8 + 2 * e + 1], dacc);
            const uint32_t hh = pack_bf16x2(p0, p1);
            hi[h * 4 + e] = hh;
            lo[h * 4 + e] = pack_bf16x2(p0 - bf16_lo_to_f32(hh), p1 - bf16_hi_to_f32(hh));
          }
        }
        // TMEM column c holds elements (2c, 2c+1) of the row: hi at [0, D/2), lo at [D/2, D)
        tmem_st16(lane_addr + C::kColPhi + half * (HD / 2) + g * 16, hi);
        tmem_st16(lane_addr + C::kColPhi + D / 2 + half * (HD / 2) + g * 16, lo);
      }
      // state rows: thread (k, half) converts S[bh][k][half*D/2 .. +D/2) into MN-major bf16
      // hi/lo tiles over the idle rings
      if (row < D) {
        const float* srow = p.S + (static_cast<size_t>(bh) * D + row) * D;
        uint8_t* s_hi = kring;
        uint8_t* s_lo = kring + D * D * 2;
#pragma unroll 4
        for (int u = 0; u < HD / 8; ++u) {
          const int unit = half * (HD / 8) + u;
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
      // combine the two halves' partial denominators and row sums
      xend[0][half][row] = dacc;
      xend[1][half][row] = l_run;
      mbar_arrive(pair_bar);  // the pair barrier's only phase
      ok = __all_sync(0xffffffffu, mbar_wait(pair_bar, 0, abort_flag, p.timeout_ns, (kKernAttn << 8) | 18));
      den = dacc + xend[0][half ^ 1][row] + 1e-6f;
      l_tot = l_run + xend[1][half ^ 1][row];
    }

    // ---- epilogue: O = O_s / l + O_lin / den -> bf16 -> TMA store of the block's rows
    ok = ok && mbar_wait(&lin_bar, 0, abort_flag, p.timeout_ns, (kKernAttn << 8) | 13);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      tc_fence_after();
      const float inv_l = (j > 0 && l_tot > 0.f) ? 1.0f / l_tot : 0.0f;
      const float inv_den = 1.0f / den;
#pragma unroll
      for (int c = 0; c < HD; c += 32) {
        uint32_t o[32], lin[32];
        tmem_ld32(lane_addr + C::kColO + half * HD + c, o);
        tmem_ld32(lane_addr + C::kColLin + half * HD + c, lin);
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
            const int unit = (half * HD + c) / 8 + u;
            const uint32_t off = (unit / 8) * (BLK * 128) + row * 128 + (((unit % 8) ^ (row & 7)) * 16);
            *reinterpret_cast<uint4*>(sQ + off) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
      fence_proxy_async_smem();
    }
    named_bar_sync(1, 256);
    if (ok && threadIdx.x == 128) {
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

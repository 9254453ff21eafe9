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
// block < 128 the remaining rows are computed but never stored). The kept blocks are
// dealt alternately to two softmax pipelines A and B (positions 0, 2, 4, ... and
// 1, 3, 5, ...), each with its own S buffer, O accumulator and running max / sum; the
// two partial results merge after the last block, as two online-softmax states do. While
// one pipeline exponentiates, the tensor cores run the other's MMAs, so the softmax of
// a block only has to fit within the MMAs of two blocks.
// 384 threads, three warpgroups; setmaxnreg moves registers from the first to the others:
//   warp 0      TMA producer of the Q tile (once) and of the K tile of each kept block J
//               into a ring of K slots (row coordinate J*block; rows past Nk are
//               zero-filled); warp 3 frees a K slot once its QK^T is done.
//   warp 1      TMEM owner (512 columns) + single-thread tcgen05 MMA issuer: one wait
//               (P ready) and one commit (the next S of that pipeline) per kept block, as
//               the tensor core's shallow instruction queue idles whenever it does more.
//   warp 2      TMA producer of the V tiles into a ring of V slots.
//   warp 3      ring bookkeeping, off the softmax threads' path: in kept-block order it
//               waits for S of block v (so QK(v), and PV(v-2) before it, are done), frees
//               their K and V slots, waits for V(v) and K(v+2) to land, and adds its arrival
//               to pipeline v%2's P-ready barrier (which also counts one arrival per softmax
//               warp of that pipeline).
//   warps 4..7  pipeline A, warps 8..11 pipeline B: one thread per query row (TMEM lane
//               quarter = warp % 4), the whole row of S per thread.
// TMEM columns: S_A [0,128), S_B [128,256), O_A [256,256+d), O_B [384,384+d). P (bf16
// pairs) overwrites the first block/2 columns of its S buffer once S is in registers.
// MMA order: S_A0 S_B0 | PV_A0 S_A1 | PV_B0 S_B1 | PV_A1 S_A2 | ...; the commit after
// S_p(i+1) also covers PV_p(i), so a softmax thread that sees S_p(i+1) knows O_p is
// stable (its lazy rescale needs no other wait).
// Softmax: online in the log2 domain with a lazily raised running max (O is rescaled only
// when a block maximum exceeds the running max by more than 8, i.e. a factor 256; exact
// since numerator and denominator share the max); the O rescale is warp-uniform because
// TMEM access is warp-collective; exp2 runs on MUFU (ex2.approx).
// Temporal RoPE variant (kRope, hf_hybrid_attn_fwd_rope; Hybrid Forcing, German technical
// summary section 2 C): a fourth warpgroup (warps 12..15, one thread per row) builds a
// table of (cos, sin) for every index 0..cap and pair, turns the Q tile's first 64
// columns into a separate buffer (the MMAs read it in place of Q's chunk 0; the raw Q
// stays for the readout) and every kept K tile in place once it has landed (dimensions
// [0, d_t), pairs (2i, 2i+1), the index of the row's frame); the MMA issuer and warp 3
// wait for "turned" in place of "landed". The rings lose one V slot to make room.
// Linear term, after the last block: phi(q) in fp32 split into bf16 hi + lo (TMEM, over
// S_B); the state's S as bf16 hi + lo comes from the split copy kept beside the state
// (bulk copies into the idle K ring, issued by the MMA thread once the last MMAs are done);
// D_lin = phi_hi S_hi + phi_hi S_lo + phi_lo S_hi on the tensor cores (TMEM, over S_A),
// denominator phi(q).z + 1e-6 in fp32; the epilogue writes
// (w_A O_A + w_B O_B) / (w_A l_A + w_B l_B) + D_lin / den, w_p = 2^(m_p - max(m_A, m_B)).
#pragma once

#include "hf_ptx.cuh"

namespace hf {

constexpr uint32_t kKernAttn = 3;
constexpr int kAttnThreads = 384;
constexpr int kAttnThreadsRope = 512;  // + the RoPE warpgroup
constexpr int kRegsSupport = 104;   // registers per thread, producer/MMA warpgroup
constexpr int kRegsSupportRope = 56;  // producer/MMA and RoPE warpgroups, with the RoPE warpgroup
constexpr int kRegsRows = 200;     // registers per thread, softmax warpgroups
static_assert(128 * kRegsSupport + 256 * kRegsRows <= kAttnThreads * 168, "setmaxnreg split exceeds the launch");
static_assert(2 * 128 * kRegsSupportRope + 256 * kRegsRows <= kAttnThreadsRope * 128,
              "setmaxnreg split exceeds the launch");
constexpr int kSmemLimit = 232448;  // max shared memory per CTA on sm_100
constexpr int kAttnStaticSmem = 1024;  // upper bound of the kernel's static shared memory
constexpr int kMaxSlots = 6;
constexpr int kSplitCopyBytes = 32 * 1024;  // bytes per bulk copy of the state's split tiles

template <int D, int BLK, bool kRope = false>
struct AttnCfg {
  static constexpr int kChunks = D / 64;
  static constexpr int kQBytes = 128 * D * 2;
  static constexpr int kQRotBytes = kRope ? 128 * 128 : 0;   // the Q tile's first 64 columns, turned
  static constexpr int kTabBytes = kRope ? 64 * 32 * 8 : 0;  // (cos, sin) of index 0..63 x pair 0..31
  static constexpr int kKVTileBytes = BLK * D * 2;
  static constexpr int kReadoutBytes = 2 * D * D * 2;  // S_hi + S_lo (bf16, d x d each)
  static constexpr int kXchBytes = 3 * 2 * 128 * 4;    // end-of-tile exchange [m | l | den][pipe][row]
  static constexpr int kTiles =
      (kSmemLimit - kAttnStaticSmem - 1024 - kQBytes - kQRotBytes - kTabBytes) / kKVTileBytes;
  static constexpr int kKSlots = ((kTiles + 1) / 2) < kMaxSlots ? ((kTiles + 1) / 2) : kMaxSlots;
  static constexpr int kVSlots = (kTiles - kKSlots) < kMaxSlots ? (kTiles - kKSlots) : kMaxSlots;
  static_assert(kKSlots >= 2 && kVSlots >= 2, "ring too small");
  static_assert(kReadoutBytes + kXchBytes <= (kKSlots + kVSlots) * kKVTileBytes,
                "readout operands and the exchange must fit in the rings");
  static constexpr int kDynSmem = 1024 + kQBytes + kQRotBytes + kTabBytes + (kKSlots + kVSlots) * kKVTileBytes;
  static_assert(kDynSmem + kAttnStaticSmem <= kSmemLimit, "shared memory");
  static constexpr uint32_t kColS = 0;      // S_A at 0, S_B at 128
  static constexpr uint32_t kColO = 256;    // O_A at 256, O_B at 384
  static constexpr uint32_t kColLin = 0;    // linear term (after the last block)
  static constexpr uint32_t kColPhi = 128;  // phi(q) hi | lo (after the last block)
  static constexpr int kHD = D / 2;         // output / phi columns per pipeline thread at the end
};

struct AttnParams {
  const int32_t* idx;  // [BH][nQB][r]
  const uint8_t* S_split;  // [BH][hi | lo tile]: the state S split into two bf16 terms
  const float* z;      // [BH][D]
  int nQB, nKB, r;
  int last_len;        // valid tokens of key block nKB - 1
  float scale_log2;    // softmax scale * log2(e)
  unsigned long long timeout_ns;
  int inject;          // test only: the first S-ready commit is skipped
  // temporal RoPE (kRope): rotated dimensions [0, rope_dt), frames of rope_T tokens, Q's
  // first token in window frame q_frame0, n_frames window frames, index cap
  int rope_dt, rope_T, q_frame0, n_frames, rope_cap;
  float rope_log2base;
};

template <int D, int BLK, bool kRope = false>
__global__ void __launch_bounds__(kRope ? kAttnThreadsRope : kAttnThreads, 1)
    hybrid_attn_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
                       const __grid_constant__ CUtensorMap mapV, const __grid_constant__ CUtensorMap mapO,
                       AttnParams p) {
  using C = AttnCfg<D, BLK, kRope>;
  constexpr int NSK = C::kKSlots;
  constexpr int NSV = C::kVSlots;
  constexpr int HD = C::kHD;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                             // Q tile; reused as the output staging tile
  uint8_t* qrot = sQ + C::kQBytes;                 // kRope: the Q tile's first chunk, turned
  uint8_t* rtab = qrot + C::kQRotBytes;            // kRope: (cos, sin) table
  uint8_t* kring = rtab + C::kTabBytes;            // NSK K slots
  uint8_t* vring = kring + NSK * C::kKVTileBytes;  // NSV V slots (S_hi/S_lo + exchange over both rings at the end)

  __shared__ uint64_t q_bar, kfull_bar[NSK], kempty_bar[NSK], vfull_bar[NSV], vempty_bar[NSV];
  __shared__ uint64_t sfull_bar[2], pfull_bar[2], final_bar, pro_bar, lin_bar, drain_bar, split_bar;
  __shared__ uint64_t qrot_bar, krot_bar[NSK];  // kRope: the Q tile / K slot has been turned
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int bh = blockIdx.x / p.nQB;
  const int I = blockIdx.x % p.nQB;
  const int32_t* idx_row = p.idx + (static_cast<size_t>(bh) * p.nQB + I) * p.r;
  volatile int* abort_flag = &abort_sh;

  if (threadIdx.x == 0) {
    mbar_init(&q_bar, 1);
    for (int s = 0; s < NSK; ++s) {
      mbar_init(&kfull_bar[s], 1);
      mbar_init(&kempty_bar[s], 1);
    }
    for (int s = 0; s < NSV; ++s) {
      mbar_init(&vfull_bar[s], 1);
      mbar_init(&vempty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sfull_bar[b], 1);
      mbar_init(&pfull_bar[b], 5);  // the pipeline's 4 warps + warp 3
    }
    mbar_init(&final_bar, 1);
    mbar_init(&split_bar, 1);
    mbar_init(&pro_bar, 8);  // the 8 softmax warps
    mbar_init(&lin_bar, 1);
    mbar_init(&drain_bar, 1);
    mbar_init(&qrot_bar, 4);  // the RoPE warpgroup's 4 warps
    for (int s = 0; s < NSK; ++s) mbar_init(&krot_bar[s], 4);
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
  // Q, K, V, idx, S and z may come from the previous grid of the stream; the next grid may
  // be scheduled once every CTA of this one has started (it then fills the SMs that this
  // grid's last CTAs leave)
  griddep_wait();
  griddep_launch_dependents();

  // With RoPE the Q tile's chunk 0 is read from qrot and a K slot only once turned.
  uint64_t* q_ready = kRope ? &qrot_bar : &q_bar;
  uint64_t* k_ready = kRope ? krot_bar : kfull_bar;

  if (warp < 4) {
   // warpgroup 0: producers and MMA issuer give registers to the softmax warpgroups
   warpgroup_reg_dec<kRope ? kRegsSupportRope : kRegsSupport>();
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
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, BLK, false, false);  // A=Q, B=K: both K-major
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
      const uint64_t qdesc = sdesc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t qrdesc = sdesc_sw128(smem_u32(qrot), 16, 1024);
      const uint64_t kdesc = sdesc_sw128(smem_u32(kring), 16, 1024);
      const uint64_t vdesc = sdesc_sw128(smem_u32(vring), BLK * 128, 1024);
      // The tensor core's instruction queue is shallow: whatever this thread does between
      // MMAs leaves it idle. So each kept block costs one wait and one commit here; the
      // slot releases and the K / V arrival checks are done by warp 3.
      // S of kept block v (valid position) into the S buffer of pipeline v % 2
      auto qk = [&](int v) {
        const uint64_t kd = kdesc + static_cast<uint64_t>(((v % NSK) * C::kKVTileBytes) >> 4);
        const uint32_t d_tmem = tmem + C::kColS + (v & 1) * 128;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          constexpr int kQChunk = (128 * 128) >> 4;
          constexpr int kKChunk = (BLK * 128) >> 4;
          const uint64_t qa = (kRope && ks < 4) ? qrdesc + (ks % 4) * 2 : qdesc + (ks / 4) * kQChunk + (ks % 4) * 2;
          umma_ss(d_tmem, qa, kd + (ks / 4) * kKChunk + (ks % 4) * 2, idesc_qk, ks > 0 ? 1u : 0u);
        }
      };
      // O_p += P_p V for kept block v, p = v % 2 (P over the first columns of S_p)
      auto pv = [&](int v) {
        const int pp = v & 1;
        const uint64_t vd = vdesc + static_cast<uint64_t>(((v % NSV) * C::kKVTileBytes) >> 4);
        const uint32_t o_tmem = tmem + C::kColO + pp * 128;
        const uint32_t p_tmem = tmem + C::kColS + pp * 128;
#pragma unroll
        for (int ks = 0; ks < BLK / 16; ++ks)
          umma_ts(o_tmem, p_tmem + ks * 8, vd + ks * 128, idesc_pv, (v > 1 || ks > 0) ? 1u : 0u);
      };
      bool ok = mbar_wait(q_ready, 0, abort_flag, p.timeout_ns, (kKernAttn << 8) | 4);
      for (int v = 0; v < 2 && v < n && ok; ++v) {
        if ((ok = mbar_wait(&k_ready[v], 0, abort_flag, p.timeout_ns, (kKernAttn << 8) | 6))) {
          tc_fence_after();
          qk(v);
          if (!(p.inject && v == 0)) umma_commit(&sfull_bar[v]);
        }
      }
      for (int v = 0; v < n && ok; ++v) {
        // P_p(i) written, V(v) and K(v+2) landed (checked by warp 3)
        if (!(ok = mbar_wait(&pfull_bar[v & 1], (v >> 1) & 1, abort_flag, p.timeout_ns, (kKernAttn << 8) | 7)))
          break;
        tc_fence_after();
        pv(v);
        // S_p(i+1) overwrites P_p(i): issued after PV_p(i), which the tensor core runs first;
        // its commit also tells pipeline p that PV_p(i) is done (O_p stable, V slot free)
        if (v + 2 < n) {
          qk(v + 2);
          umma_commit(&sfull_bar[v & 1]);
        }
      }
      if (ok) {
        umma_commit(&final_bar);
        // once every MMA is done the K ring is idle: the state's hi and lo tiles, kept beside
        // the state in the readout MMAs' layout, go into it by bulk copies
        bool copying = false;
        if ((ok = mbar_wait(&final_bar, 0, abort_flag, p.timeout_ns, (kKernAttn << 8) | 9))) {
          const uint8_t* src = p.S_split + static_cast<size_t>(bh) * C::kReadoutBytes;
          mbar_arrive_expect_tx(&split_bar, C::kReadoutBytes);
          for (int o = 0; o < C::kReadoutBytes; o += kSplitCopyBytes)
            bulk_load(kring + o, src + o, min(kSplitCopyBytes, C::kReadoutBytes - o), &split_bar);
          copying = true;
        }
        // linear term: D_lin = phi_hi S_hi + phi_hi S_lo + phi_lo S_hi
        if (ok && (ok = mbar_wait(&pro_bar, 0, abort_flag, p.timeout_ns, (kKernAttn << 8) | 5)) &&
            (ok = mbar_wait(&split_bar, 0, abort_flag, p.timeout_ns, (kKernAttn << 8) | 16))) {
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
        if (copying) mbar_wait_drain(&split_bar, 0, p.timeout_ns, (kKernAttn << 8) | 16);
      }
      umma_commit(&drain_bar);
      mbar_wait_drain(&drain_bar, 0, p.timeout_ns, (kKernAttn << 8) | 8);
    }
   } else {
    // ============================ ring bookkeeping ============================
    if (lane == 0) {
      int n = 0;
      for (int jj = 0; jj < p.r; ++jj) {
        const int J = __ldg(idx_row + jj);
        n += (J >= 0 && J < p.nKB);
      }
      // Every barrier below is waited on phase after phase, in order, by this one thread,
      // so a parity wait can never be satisfied by an older phase.
      for (int v = 0; v < n; ++v) {
        const int pp = v & 1, i = v >> 1;
        // S_p(i) done: QK(v) has read K(v); PV(v-2), committed before it, has read V(v-2).
        // (P-ready phase i-1 of this pipeline is therefore complete too.)
        if (!mbar_wait(&sfull_bar[pp], i & 1, abort_flag, p.timeout_ns, (kKernAttn << 8) | 17)) break;
        mbar_arrive(&kempty_bar[v % NSK]);
        if (i > 0) mbar_arrive(&vempty_bar[(v - 2) % NSV]);
        // the MMA issuer runs PV(v) and QK(v+2) on P-ready: their tiles must be there
        if (!mbar_wait(&vfull_bar[v % NSV], (v / NSV) & 1, abort_flag, p.timeout_ns, (kKernAttn << 8) | 14)) break;
        if (v + 2 < n &&
            !mbar_wait(&k_ready[(v + 2) % NSK], ((v + 2) / NSK) & 1, abort_flag, p.timeout_ns, (kKernAttn << 8) | 15))
          break;
        mbar_arrive(&pfull_bar[pp]);
      }
    }
   }
  } else if (warp >= 12) {
    // ============== temporal RoPE warpgroup: turns the Q tile and every kept K tile ==============
    warpgroup_reg_dec<kRegsSupportRope>();
    if constexpr (kRope) {
      const int rt = threadIdx.x - 384;  // a row of the Q tile, or of a K tile
      const int npair = p.rope_dt / 2;
      const int nunits = (p.rope_dt + 7) / 8;  // 16-byte units of chunk 0 that hold turned pairs
      float2* tab = reinterpret_cast<float2*>(rtab);  // [index][pair]
      for (int e = rt; e < (p.rope_cap + 1) * 32; e += 128) {
        const int pi = e / 32, i = e % 32;
        float c = 1.f, sn = 0.f;
        if (i < npair) {
          const float theta = exp2f(-static_cast<float>(2 * i) / static_cast<float>(p.rope_dt) * p.rope_log2base);
          sincosf(static_cast<float>(pi) * theta, &sn, &c);
        }
        tab[e] = make_float2(c, sn);
      }
      named_bar_sync(2, 128);
      // index of window frame w (newest at the cap); padding rows clamp into the table
      auto index_of = [&](int w) { return min(max(p.rope_cap - min((p.n_frames - 1) - w, p.rope_cap), 0), p.rope_cap); };
      // units [0, nunits) of one 128-byte row of a 128B-swizzled chunk turned from src to dst,
      // units [nunits, nall) copied
      auto turn_row = [&](const uint8_t* src, uint8_t* dst, int row, int pidx, int nall) {
        const float2* trow = tab + pidx * 32;
        for (int u = 0; u < nall; ++u) {
          const uint32_t off = row * 128 + ((u ^ (row & 7)) * 16);
          const uint4 w = *reinterpret_cast<const uint4*>(src + off);
          uint32_t ww[4] = {w.x, w.y, w.z, w.w};
          if (u < nunits) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int i = 4 * u + e;
              if (i < npair) {
                const float x0 = bf16_lo_to_f32(ww[e]), x1 = bf16_hi_to_f32(ww[e]);
                const float2 cs = trow[i];
                ww[e] = pack_bf16x2(fmaf(x0, cs.x, -x1 * cs.y), fmaf(x0, cs.y, x1 * cs.x));
              }
            }
          }
          *reinterpret_cast<uint4*>(dst + off) = make_uint4(ww[0], ww[1], ww[2], ww[3]);
        }
      };
      // the Q tile: chunk 0 into qrot (every unit, the first nunits turned)
      bool ok = mbar_wait(&q_bar, 0, abort_flag, p.timeout_ns, (kKernAttn << 8) | 20);
      if (ok) {
        const int tok = I * BLK + rt;  // token of the chunk (rows past Nq hold TMA zeros)
        turn_row(sQ, qrot, rt, index_of(p.q_frame0 + tok / p.rope_T), 8);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&qrot_bar);
      }
      // every kept K tile, in place, in kept-block order
      int v = 0;
      for (int jj = 0; jj < p.r && ok; ++jj) {
        const int J = __ldg(idx_row + jj);
        if (J < 0 || J >= p.nKB) continue;
        const int s = v % NSK;
        ok = mbar_wait(&kfull_bar[s], (v / NSK) & 1, abort_flag, p.timeout_ns, (kKernAttn << 8) | 21);
        if (!ok) break;
        // rows at index 0 (frames at least cap frames old) are left as they are: the
        // rotation is the identity there
        const bool valid = rt < BLK && (J < p.nKB - 1 || rt < p.last_len);
        const int pidx = index_of((J * BLK + rt) / p.rope_T);
        if (valid && pidx > 0) {
          uint8_t* ktile = kring + s * C::kKVTileBytes;  // chunk 0: BLK rows x 128 B
          turn_row(ktile, ktile, rt, pidx, nunits);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&krot_bar[s]);
        ++v;
      }
    }
  } else {
    warpgroup_reg_inc<kRegsRows>();
    // ======================= softmax pipelines, readout, epilogue =======================
    const int quarter = warp & 3;
    const int pipe = (warp - 4) >> 2;     // 0: warps 4..7 (A), 1: warps 8..11 (B)
    const int row = quarter * 32 + lane;  // query row within the tile == TMEM lane
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const uint32_t col_s = C::kColS + pipe * 128;
    const uint32_t col_o = C::kColO + pipe * 128;
    bool ok = true;

    // ---- online softmax over this pipeline's kept blocks (the whole row per thread)
    float m_run = -INFINITY, l_run = 0.f;
    int v = 0, i = 0;  // valid kept position, blocks of this pipeline so far
    for (int jj = 0; jj < p.r && ok; ++jj) {
      const int J = __ldg(idx_row + jj);
      if (J < 0 || J >= p.nKB) continue;
      if ((v++ & 1) != pipe) continue;
      // tcgen05.ld/st are warp-collective: every wait that guards one is made warp-uniform
      ok = __all_sync(0xffffffffu, mbar_wait(&sfull_bar[pipe], i & 1, abort_flag, p.timeout_ns,
                                             (kKernAttn << 8) | 10));
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[BLK];
      tmem_ld_cols<BLK>(lane_addr + col_s, sr);
      tmem_wait_ld();
      reg_fence<BLK>(sr);
      float* srow = reinterpret_cast<float*>(sr);
      const int valid = (J == p.nKB - 1) ? p.last_len : BLK;
      if (valid < BLK) {  // partial last key block: padding columns are masked out
#pragma unroll
        for (int c = 0; c < BLK; ++c)
          if (c >= valid) srow[c] = -INFINITY;
      }
      // row max: independent chains of 3-input max
      constexpr int kMC = BLK >= 64 ? 8 : 4;
      float mc[kMC];
#pragma unroll
      for (int k = 0; k < kMC; ++k) mc[k] = fmaxf(srow[k], srow[k + kMC]);
#pragma unroll
      for (int c = 2 * kMC; c < BLK; c += 2 * kMC) {
#pragma unroll
        for (int k = 0; k < kMC; ++k) mc[k] = fmax3(mc[k], srow[c + k], srow[c + kMC + k]);
      }
      float mx = mc[0];
#pragma unroll
      for (int k = 1; k < kMC; ++k) mx = fmaxf(mx, mc[k]);
      mx *= p.scale_log2;
      // A row raises its running max only when the block max exceeds it by more than 8
      // (log2 units); O_p and l are then scaled by alpha = 2^(m_old - m_new).
      float alpha = 1.0f;
      const bool need = i > 0 && mx > m_run + 8.0f;
      if (i == 0) {
        m_run = mx;
      } else if (need) {
        alpha = ex2_approx(m_run - mx);
        l_run *= alpha;
        m_run = mx;
      }
      // p = 2^(s * scale * log2 e - m): scale and shift as packed fp32 pairs, exp2 on MUFU,
      // 32 columns at a time; each chunk of P goes to TMEM over the first columns of S_p at
      // once (S is in registers). The softmax warps share their SM sub-partitions with the
      // MMA-issuing thread, so fewer instructions per element matter more than spreading
      // exp2 over the FMA pipe (a polynomial exp2 costs ~6x the issue slots of MUFU's).
      {
        const uint64_t sl2 = f32x2(p.scale_log2, p.scale_log2);
        const uint64_t nm2 = f32x2(-m_run, -m_run);
        uint64_t lacc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int c0 = 0; c0 < BLK; c0 += 32) {
          uint32_t pk[16];
#pragma unroll
          for (int c = c0; c < c0 + 32; c += 2) {
            float x0, x1;
            f32x2_split(ffma2(f32x2(srow[c], srow[c + 1]), sl2, nm2), x0, x1);
            const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
            lacc[(c / 2) & 3] = fadd2(lacc[(c / 2) & 3], f32x2(p0, p1));
            pk[(c - c0) / 2] = pack_bf16x2(p0, p1);
          }
          tmem_st16(lane_addr + col_s + c0 / 2, pk);
        }
        const uint64_t l2 = fadd2(fadd2(lacc[0], lacc[1]), fadd2(lacc[2], lacc[3]));
        float la, lb;
        f32x2_split(l2, la, lb);
        l_run += la + lb;
      }
      // lazy O rescale, by the whole warp whenever any of its rows needs it (alpha = 1 for
      // the others); O_p is stable: PV_p(i-1) completed before S_p(i) was signalled
      if (__any_sync(0xffffffffu, need)) {
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          uint32_t o[32];
          tmem_ld32(lane_addr + col_o + c, o);
          tmem_wait_ld();
          reg_fence<32>(o);
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
          tmem_st32(lane_addr + col_o + c, o);
        }
      }
      // one arrival per warp, once every lane's P (and O rescale) stores are complete
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&pfull_bar[pipe]);
      ++i;
    }

    // ---- linear term operands. This thread's half of z does not depend on the MMAs: its
    // loads are issued before the wait for the last MMAs, so that their latency hides behind
    // it. (The state's hi and lo tiles arrive in the K ring by the MMA thread's bulk copies.)
    constexpr int kQ4 = HD / 4;  // float4 per half row
    float4 zv[kQ4];
    {
      const float4* z4 = reinterpret_cast<const float4*>(p.z + static_cast<size_t>(bh) * D + pipe * HD);
#pragma unroll
      for (int k = 0; k < kQ4; ++k) zv[k] = __ldg(z4 + k);
    }
    // (all MMAs done: the S buffers and both rings are free)
    ok = ok && mbar_wait(&final_bar, 0, abort_flag, p.timeout_ns, (kKernAttn << 8) | 12);
    ok = __all_sync(0xffffffffu, ok);
    float dacc = 0.f;
    if (ok) {
      tc_fence_after();
      // phi(x) = max(x, 0) + 2^(min(x, 0) log2 e) (branch-free elu + 1) on packed fp32 pairs;
      // phi . z accumulated as a pair, summed at the end
      uint64_t dacc2 = 0ull;
#pragma unroll
      for (int g = 0; g < HD / 32; ++g) {  // 32 elements -> 16 packed columns of hi and of lo
        uint32_t hi[16], lo[16];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const int unit = pipe * (HD / 8) + g * 4 + h;  // elements [8*unit, 8*unit + 8)
          const uint32_t off = (unit / 8) * (128 * 128) + row * 128 + (((unit % 8) ^ (row & 7)) * 16);
          const uint4 qv = *reinterpret_cast<const uint4*>(sQ + off);
          const float4 za = zv[(g * 4 + h) * 2], zb = zv[(g * 4 + h) * 2 + 1];
          const uint32_t w[4] = {qv.x, qv.y, qv.z, qv.w};
          const uint64_t zz[4] = {f32x2(za.x, za.y), f32x2(za.z, za.w), f32x2(zb.x, zb.y), f32x2(zb.z, zb.w)};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float x0 = bf16_lo_to_f32(w[e]), x1 = bf16_hi_to_f32(w[e]);
            const float n0 = fminf(x0, 0.f), n1 = fminf(x1, 0.f);
            float l0, l1;
            f32x2_split(ffma2(f32x2(n0, n1), f32x2(1.4426950408889634f, 1.4426950408889634f), 0ull), l0, l1);
            // (x - min(x, 0)) + 2^l
            const uint64_t p2 = fadd2(ffma2(f32x2(n0, n1), f32x2(-1.0f, -1.0f), f32x2(x0, x1)),
                                      f32x2(ex2_approx(l0), ex2_approx(l1)));
            dacc2 = ffma2(p2, zz[e], dacc2);
            float p0, p1;
            f32x2_split(p2, p0, p1);
            const uint32_t hh = pack_bf16x2(p0, p1);
            hi[h * 4 + e] = hh;
            float r0, r1;
            f32x2_split(ffma2(f32x2(bf16_lo_to_f32(hh), bf16_hi_to_f32(hh)), f32x2(-1.0f, -1.0f), p2), r0, r1);
            lo[h * 4 + e] = pack_bf16x2(r0, r1);
          }
        }
        // TMEM column c holds elements (2c, 2c+1) of the row: hi at [0, D/2), lo at [D/2, D)
        tmem_st16(lane_addr + C::kColPhi + pipe * (HD / 2) + g * 16, hi);
        tmem_st16(lane_addr + C::kColPhi + D / 2 + pipe * (HD / 2) + g * 16, lo);
      }
      {
        float d0, d1;
        f32x2_split(dacc2, d0, d1);
        dacc = d0 + d1;
      }
      fence_proxy_async_smem();
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&pro_bar);
    }
    // ---- merge of the two pipelines' softmax states and denominators (every row thread
    // reaches both named barriers, whatever happened before)
    float* xch = reinterpret_cast<float*>(kring + C::kReadoutBytes);  // [3][2][128]
    xch[(0 * 2 + pipe) * 128 + row] = m_run;
    xch[(1 * 2 + pipe) * 128 + row] = l_run;
    xch[(2 * 2 + pipe) * 128 + row] = dacc;
    named_bar_sync(1, 256);
    const float m_a = xch[(0 * 2 + 0) * 128 + row], m_b = xch[(0 * 2 + 1) * 128 + row];
    const float l_a = xch[(1 * 2 + 0) * 128 + row], l_b = xch[(1 * 2 + 1) * 128 + row];
    const float den = xch[(2 * 2 + 0) * 128 + row] + xch[(2 * 2 + 1) * 128 + row] + 1e-6f;
    // a pipeline without blocks has m = -inf: weight 0, and its O (never written) unused
    const float m_tot = fmaxf(m_a, m_b);
    const bool has_a = m_a > -INFINITY, has_b = m_b > -INFINITY;
    const float w_a = has_a ? ex2_approx(m_a - m_tot) : 0.f;
    const float w_b = has_b ? ex2_approx(m_b - m_tot) : 0.f;
    const float l_tot = (has_a ? l_a * w_a : 0.f) + (has_b ? l_b * w_b : 0.f);
    const float inv_l = l_tot > 0.f ? 1.0f / l_tot : 0.0f;
    const float inv_den = 1.0f / den;

    // ---- epilogue: this thread's half of the columns of
    // O = (w_A O_A + w_B O_B) / l + O_lin / den -> bf16 -> TMA store of the block's rows
    ok = ok && mbar_wait(&lin_bar, 0, abort_flag, p.timeout_ns, (kKernAttn << 8) | 13);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      tc_fence_after();
      const float sa = w_a * inv_l, sb = w_b * inv_l;
#pragma unroll
      for (int c = 0; c < HD; c += 32) {
        const uint32_t col = pipe * HD + c;
        uint32_t oa[32], ob[32], lin[32];
        tmem_ld32(lane_addr + C::kColO + col, oa);
        tmem_ld32(lane_addr + C::kColO + 128 + col, ob);
        tmem_ld32(lane_addr + C::kColLin + col, lin);
        tmem_wait_ld();
        reg_fence<32>(oa);
        reg_fence<32>(ob);
        reg_fence<32>(lin);
        if (row < BLK) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {  // four 16-byte units of 8 columns
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              float y[2];
#pragma unroll
              for (int t = 0; t < 2; ++t) {
                const int k = u * 8 + 2 * e + t;
                const float s_a = has_a ? __uint_as_float(oa[k]) * sa : 0.f;
                const float s_b = has_b ? __uint_as_float(ob[k]) * sb : 0.f;
                y[t] = (s_a + s_b) + __uint_as_float(lin[k]) * inv_den;
              }
              w[e] = pack_bf16x2(y[0], y[1]);
            }
            const int unit = col / 8 + u;
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

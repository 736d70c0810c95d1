// Block-sparse attention forward for sm_100a (tcgen05 + TMEM + TMA).
//
// What it computes (CalibAtt abstract and Fig. 5(b): compute the selected
// block connections exactly and skip the unselected ones; RECAP section 4.1:
// block-sparse attention for the selected interactions, dense attention for
// refreshes; RECAP section 1: a cached dense refinement corrects the sparse
// output): for every query row r of query block i,
//     O[r] = softmax over the keys of the kept blocks K(i) of (q_r.k_c/sqrt(D)) . V
//     LSE[r] = log-sum-exp of those logits,
// optionally followed by O <- O + alpha_h * R in the epilogue.
//
// Work decomposition.  A CTA owns a PAIR of 128-row query tiles of one
// (batch, head).  The two tiles usually keep overlapping key blocks (their
// queries are neighbours in token order), so the CTA walks the UNION of the
// kept lists of its query blocks in ascending key-block order and loads each
// K/V block once for both tiles; each tile only computes the blocks it keeps.
// With blk = 64 one 128-row tile spans two query blocks; rows of the half that
// does not keep a block are masked to -inf for that block.
//
// Half blocks.  Scores are produced and consumed in 64-key halves, and every
// tile has two S buffers in TMEM, so the tensor core computes S for half h+1
// (and h+2) while the softmax works on half h: a tile never waits for its own
// PV -> S round trip.  P of half h (bf16 pairs) overwrites the first 32
// columns of its S buffer; S of half h+2 reuses the buffer only after the PV
// of half h has completed.
//
// Warp roles (16 warps):
//   warp 0        TMA: Q (once), then K of every union entry (ring of NSK)
//   warp 1        TMA: V of every union entry (ring of NSV)
//   warp 2 / 12   S issuer of tile 0 / 1: S_h = Q K_h^T, K-major operands in
//                 shared memory, fp32 accumulator in TMEM
//   warp 3 / 13   PV issuer of tile 0 / 1: O += P_h V_h, P from TMEM, V
//                 MN-major in shared memory
//   warp 14       TMEM allocation
//   warps 4-7     softmax + epilogue of tile 0 (one thread per query row)
//   warps 8-11    softmax + epilogue of tile 1
// TMEM columns: S0a S0b | S1a S1b | O0 | O1.
//
// Every issuer walks the union in order and waits on every entry's landing,
// member or not: a parity wait cannot tell phase k of a barrier from phase
// k-2, so a thread that skipped entries could take an older phase for the one
// it wants.  For an entry its tile does not keep, an issuer releases the slot
// with a plain arrive, so each release barrier gets exactly one arrival per
// issuer of that ring (two) and entry.
//
// Online softmax in the log2 domain in fp32.  The running max used for the
// exponentials is only raised when a half-block max exceeds it by more than 8
// (so P <= 2^8); O in TMEM is rescaled only then (after the previous PV has
// completed), and the final 1/l uses the same reference, so the result is
// exact up to rounding.
//
// Every wait is bounded (2 s of globaltimer); a timeout sets BSA_DEV_TIMEOUT
// in the caller's status word, aborts the CTA's pipeline, drains what is in
// flight and releases TMEM.
#include <cuda.h>
#include <cuda_bf16.h>

#include <cmath>
#include <cstdio>

#include "internal.cuh"
#include "sm100.cuh"

namespace bsa {
namespace {

using namespace sm100;

constexpr int kThreads = 512;
constexpr int BM = 128;                         // query rows per tile
constexpr int SN = 64;                          // keys per half block (S buffer width)
constexpr uint64_t kTimeoutNs = 2000000000ull;  // 2 s
constexpr float kRescaleThreshold = 8.0f;       // log2 units
constexpr int kRegsLaunch = 128;                // 65536 / 512
constexpr int kRegsCtl = 56;
constexpr int kRegsSoftmax = 200;
static_assert(256 * kRegsCtl + 256 * kRegsSoftmax <= kThreads * kRegsLaunch, "register split exceeds launch");

struct Params {
  const int32_t* kept_idx;
  const int32_t* kept_cnt;
  const __nv_bfloat16* R;
  const float* alpha;
  __nv_bfloat16* o;
  float* lse;
  int32_t* status;
  int H, L, NB;
  float scale_log2;
  int dense;
};

template <int D, int BN>
struct Cfg {
  static constexpr int G = BM / BN;               // query blocks per 128-row tile
  static constexpr int HB = BN / SN;              // halves per key block
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int KV_BYTES = BN * D * 2;     // one K or one V tile
  static constexpr int UNION_BYTES = kMaxNB * 2;  // uint16 per union entry
  static constexpr int MISC_BYTES = 512;          // barriers and scalars
  static constexpr int SLOTS = (227 * 1024 - 1024 - 2 * Q_BYTES - UNION_BYTES - MISC_BYTES) / KV_BYTES;
  static constexpr int NSK = ((SLOTS + 1) / 2) > 4 ? 4 : (SLOTS + 1) / 2;
  static constexpr int NSV = (SLOTS / 2) > 4 ? 4 : SLOTS / 2;
  static_assert(NSK >= 2 && NSV >= 2, "shared memory too small for double-buffered K and V");
  static_assert(KV_BYTES >= kMaxNB, "the set-up bitmap is staged in the first K slot");
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = 2 * Q_BYTES;
  static constexpr int OFF_V = OFF_K + NSK * KV_BYTES;
  static constexpr int OFF_UNION = OFF_V + NSV * KV_BYTES;
  static constexpr int OFF_MISC = OFF_UNION + UNION_BYTES;
  static constexpr int SMEM_BYTES = OFF_MISC + MISC_BYTES + 1024;  // + alignment slack
  static constexpr int COL_O = 4 * SN;                            // O_t at COL_O + t*D
  static constexpr int TMEM_COLS = 512;
  static constexpr int PANELS = D / 64;
};

struct Shared {
  // laid out in the MISC region
  uint64_t full_k[4];
  uint64_t empty_k[4];
  uint64_t full_v[4];
  uint64_t empty_v[4];
  uint64_t q_full;
  uint64_t s_full[2][2];   // [tile][buffer]
  uint64_t p_full[2][2];
  uint64_t pv_done[2][2];
  uint64_t o_full[2];
  uint64_t drain[4];
  uint32_t tmem_base;
  uint32_t n_union;
  uint32_t n_tile[2];
  volatile int abort_flag;
};
static_assert(sizeof(Shared) <= 512, "misc region too small");

__device__ __forceinline__ void flag_status(const Params& prm, int bits) {
  if (prm.status) atomicOr(prm.status, bits);
}

// Bounded blocking wait.  Returns false on timeout or when another role has
// already aborted the CTA.
__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity, Shared* sh, const Params& prm) {
  if (mbar_try(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try(bar, parity)) return true;
    if ((it & 15) == 0) {
      if (sh->abort_flag) return false;
      if (globaltimer_ns() - t0 > kTimeoutNs) {
        sh->abort_flag = 1;
        flag_status(prm, BSA_DEV_TIMEOUT);
        return false;
      }
    }
  }
}

// Warp-uniform bounded wait (every lane waits; all must succeed).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, Shared* sh, const Params& prm) {
  const bool ok = wait_bounded(bar, parity, sh, prm);
  return __all_sync(0xffffffffu, ok);
}

// Bounded wait used only while draining after an abort.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try(bar, parity) && globaltimer_ns() - t0 < kTimeoutNs) {
  }
}

__device__ __forceinline__ int next_member(const uint16_t* ulist, int i, int U, uint32_t tile_mask) {
  while (i < U && ((ulist[i] >> 12) & tile_mask) == 0) ++i;
  return i;
}

// TMA producer of one operand ring (K or V): entry u goes to slot u % NS once
// both issuers of the ring released the slot's previous entry.
template <int D, int BN, int NS>
__device__ __forceinline__ void produce_ring(const CUtensorMap* map, uint8_t* ring, uint64_t* full, uint64_t* empty,
                                             const uint16_t* ulist, int U, int bh, int lane, Shared* sh,
                                             const Params& prm) {
  using C = Cfg<D, BN>;
  int issued = 0;
  for (int u = 0; u < U; ++u) {
    const int slot = u % NS;
    if (u >= NS && !warp_wait(&empty[slot], ((u / NS) - 1) & 1, sh, prm)) break;
    if (lane == 0) {
      const int kb = ulist[u] & 0xFFF;
      uint8_t* dst = ring + slot * C::KV_BYTES;
      mbar_arrive_expect_tx(&full[slot], C::KV_BYTES);
      for (int pnl = 0; pnl < C::PANELS; ++pnl)
        tma_load_3d(dst + pnl * BN * 128, map, &full[slot], pnl * 64, kb * BN, bh);
    }
    __syncwarp();
    issued = u + 1;
  }
  if (sh->abort_flag && lane == 0) {
    // load k of a slot is issued only after release k-1, which follows the
    // issuers' observation of landing k-1: the parity below is exact
    for (int u = issued - NS < 0 ? 0 : issued - NS; u < issued; ++u) drain_wait(&full[u % NS], (u / NS) & 1);
  }
}

template <int D, int BN>
__global__ void __launch_bounds__(kThreads, 1)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const Params prm) {
  using C = Cfg<D, BN>;
  constexpr int G = C::G;
  constexpr int HB = C::HB;
  constexpr int NSK = C::NSK;
  constexpr int NSV = C::NSV;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint16_t* ulist = reinterpret_cast<uint16_t*>(smem + C::OFF_UNION);
  uint32_t* bitmap = reinterpret_cast<uint32_t*>(smem + C::OFF_K);  // set-up only
  Shared* sh = reinterpret_cast<Shared*>(smem + C::OFF_MISC);
  uint8_t* q_smem = smem + C::OFF_Q;
  uint8_t* k_ring = smem + C::OFF_K;
  uint8_t* v_ring = smem + C::OFF_V;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int pair = blockIdx.x;
  const int bh = blockIdx.y;
  const int NB = prm.NB;
  const int L = prm.L;

  // ---------------------------------------------------------------- set-up
  if (threadIdx.x == 0) {
    for (int s = 0; s < 4; ++s) {
      mbar_init(&sh->full_k[s], 1);
      mbar_init(&sh->empty_k[s], 2);
      mbar_init(&sh->full_v[s], 1);
      mbar_init(&sh->empty_v[s], 2);
      mbar_init(&sh->drain[s], 1);
    }
    mbar_init(&sh->q_full, 1);
    for (int t = 0; t < 2; ++t) {
      for (int b = 0; b < 2; ++b) {
        mbar_init(&sh->s_full[t][b], 1);
        mbar_init(&sh->p_full[t][b], 128);
        mbar_init(&sh->pv_done[t][b], 1);
      }
      mbar_init(&sh->o_full[t], 1);
    }
    sh->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 14) {
    tmem_alloc(&sh->tmem_base, C::TMEM_COLS);
    tmem_relinquish();
    tc_fence_before();
  }
  for (int i = threadIdx.x; i < (NB + 3) / 4; i += kThreads) bitmap[i] = 0u;
  __syncthreads();

  // Membership bits: bit `sub` of key block kb is set when query block
  // pair*2G + sub keeps kb.
  for (int sub = 0; sub < 2 * G; ++sub) {
    const int qb = pair * 2 * G + sub;
    if (qb >= NB) break;
    int cnt = NB;
    const int32_t* row = nullptr;
    if (!prm.dense) {
      const size_t r = static_cast<size_t>(bh) * NB + qb;
      cnt = prm.kept_cnt[r];
      if (cnt < 0 || cnt > NB) {
        if (threadIdx.x == 0) flag_status(prm, BSA_DEV_BAD_INDEX);
        cnt = cnt < 0 ? 0 : NB;
      }
      row = prm.kept_idx + r * NB;
    }
    for (int n = threadIdx.x; n < cnt; n += kThreads) {
      const int kb = prm.dense ? n : row[n];
      if (static_cast<unsigned>(kb) >= static_cast<unsigned>(NB)) {
        flag_status(prm, BSA_DEV_BAD_INDEX);
        continue;
      }
      atomicOr(&bitmap[kb >> 2], (1u << sub) << ((kb & 3) * 8));
    }
  }
  __syncthreads();
  if (warp == 0) {
    const uint32_t m0 = (1u << G) - 1u, m1 = m0 << G;
    uint32_t U = 0, c0 = 0, c1 = 0;
    for (int base = 0; base < NB; base += 32) {
      const int kb = base + lane;
      const uint32_t m = kb < NB ? (bitmap[kb >> 2] >> ((kb & 3) * 8)) & 0xFu : 0u;
      const uint32_t bal = __ballot_sync(0xffffffffu, m != 0);
      if (m) ulist[U + __popc(bal & ((1u << lane) - 1u))] = static_cast<uint16_t>(kb | (m << 12));
      U += __popc(bal);
      c0 += __popc(__ballot_sync(0xffffffffu, (m & m0) != 0));
      c1 += __popc(__ballot_sync(0xffffffffu, (m & m1) != 0));
    }
    if (lane == 0) {
      sh->n_union = U;
      sh->n_tile[0] = c0;
      sh->n_tile[1] = c1;
    }
  }
  __syncthreads();  // union list complete; the bitmap's K slot may now be overwritten
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;
  const int U = static_cast<int>(sh->n_union);
  const int ntile[2] = {static_cast<int>(sh->n_tile[0]), static_cast<int>(sh->n_tile[1])};
  const uint32_t tile_mask[2] = {(1u << G) - 1u, ((1u << G) - 1u) << G};

  if (warp < 4 || warp >= 12) {
    // Registers: the control warpgroups (TMA, MMA issue, TMEM allocation)
    // need few; the two softmax warpgroups hold score rows.
    setmaxnreg_dec<kRegsCtl>();
    if (warp == 0 && U > 0) {
      // ------------------------------------------------ TMA: Q, then K ring
      if (lane == 0) {
        int tiles_here = 0;
        for (int t = 0; t < 2; ++t)
          if ((pair * 2 + t) * BM < L) ++tiles_here;
        mbar_arrive_expect_tx(&sh->q_full, tiles_here * C::Q_BYTES);
        for (int t = 0; t < 2; ++t) {
          const int row0 = (pair * 2 + t) * BM;
          if (row0 >= L) continue;
          for (int pnl = 0; pnl < C::PANELS; ++pnl)
            tma_load_3d(q_smem + t * C::Q_BYTES + pnl * BM * 128, &tmQ, &sh->q_full, pnl * 64, row0, bh);
        }
      }
      __syncwarp();
      produce_ring<D, BN, NSK>(&tmK, k_ring, sh->full_k, sh->empty_k, ulist, U, bh, lane, sh, prm);
    } else if (warp == 1 && U > 0) {
      // ------------------------------------------------------ TMA: V ring
      produce_ring<D, BN, NSV>(&tmV, v_ring, sh->full_v, sh->empty_v, ulist, U, bh, lane, sh, prm);
    } else if ((warp == 2 || warp == 12) && U > 0) {
      // ------------------------------------------- S issuer of one tile
      const int t = warp == 2 ? 0 : 1;
      constexpr uint32_t idS = idesc_bf16_f32(BM, SN, false, false);
      const uint32_t qa = smem_u32(q_smem) + t * C::Q_BYTES;
      const uint32_t k_base = smem_u32(k_ring);
      bool ok = ntile[t] == 0 || warp_wait(&sh->q_full, 0, sh, prm);
      tc_fence_after();
      int h = 0;
      for (int u = 0; ok && u < U; ++u) {
        const int sk = u % NSK;
        if (!(ok = warp_wait(&sh->full_k[sk], (u / NSK) & 1, sh, prm))) break;
        if (((ulist[u] >> 12) & tile_mask[t]) == 0) {
          if (lane == 0) mbar_arrive(&sh->empty_k[sk]);  // not this tile's block
          continue;
        }
        for (int j = 0; j < HB; ++j, ++h) {
          const int b = h & 1;
          // S_h reuses buffer b: P_{h-2} in it must have been consumed
          if (h >= 2 && !(ok = warp_wait(&sh->pv_done[t][b], ((h - 2) >> 1) & 1, sh, prm))) break;
          tc_fence_after();
          if (lane == 0) {
            const uint32_t ka = k_base + sk * C::KV_BYTES + j * (SN * 128);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off_q = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
              const uint32_t off_k = (kk >> 2) * (BN * 128) + (kk & 3) * 32;
              mma_ss(tmem + t * 2 * SN + b * SN, sdesc_sw128(qa + off_q, 16, 1024),
                     sdesc_sw128(ka + off_k, 16, 1024), idS, kk > 0 ? 1u : 0u);
            }
            tc_commit(&sh->s_full[t][b]);
          }
          __syncwarp();
        }
        if (!ok) break;
        if (lane == 0) tc_commit(&sh->empty_k[sk]);
        __syncwarp();
      }
      if (lane == 0 && !ok) {
        tc_commit(&sh->drain[t]);
        drain_wait(&sh->drain[t], 0);
      }
      __syncwarp();
    } else if ((warp == 3 || warp == 13) && U > 0) {
      // ------------------------------------------ PV issuer of one tile
      const int t = warp == 3 ? 0 : 1;
      constexpr uint32_t idPV = idesc_bf16_f32(BM, D, false, true);
      const uint32_t v_base = smem_u32(v_ring);
      const uint32_t colO = C::COL_O + t * D;
      bool ok = true;
      int h = 0;
      for (int u = 0; ok && u < U; ++u) {
        const int sv = u % NSV;
        if (!(ok = warp_wait(&sh->full_v[sv], (u / NSV) & 1, sh, prm))) break;
        if (((ulist[u] >> 12) & tile_mask[t]) == 0) {
          if (lane == 0) mbar_arrive(&sh->empty_v[sv]);  // not this tile's block
          continue;
        }
        for (int j = 0; j < HB; ++j, ++h) {
          const int b = h & 1;
          if (!(ok = warp_wait(&sh->p_full[t][b], (h >> 1) & 1, sh, prm))) break;
          tc_fence_after();
          if (lane == 0) {
            const uint32_t va = v_base + sv * C::KV_BYTES + j * (SN * 128);
#pragma unroll
            for (int kk = 0; kk < SN / 16; ++kk)
              mma_ts(tmem + colO, tmem + t * 2 * SN + b * SN + kk * 8,
                     sdesc_sw128(va + kk * 2048, BN * 128, 1024), idPV, (h > 0 || kk > 0) ? 1u : 0u);
            tc_commit(&sh->pv_done[t][b]);
          }
          __syncwarp();
        }
        if (!ok) break;
        if (lane == 0) tc_commit(&sh->empty_v[sv]);
        __syncwarp();
      }
      if (lane == 0) {
        if (ok && h > 0) tc_commit(&sh->o_full[t]);
        if (!ok) {
          tc_commit(&sh->drain[2 + t]);
          drain_wait(&sh->drain[2 + t], 0);
        }
      }
      __syncwarp();
    }
  } else {
    // ------------------------------------------------ softmax + epilogue
    setmaxnreg_inc<kRegsSoftmax>();
    const int t = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_off + t * 2 * SN;  // + b * SN
    const uint32_t tO = tmem + lane_off + C::COL_O + t * D;
    const int grow = (pair * 2 + t) * BM + r;
    const uint32_t my_bit = 1u << (t * G + r / BN);
    const float sl2 = prm.scale_log2;
    float m_ref = -INFINITY;
    float l = 0.f;
    bool ok = true;
    int u = next_member(ulist, 0, U, tile_mask[t]);
    int h = 0;
    for (int n = 0; ok && n < ntile[t]; ++n) {
      const uint32_t e = ulist[u];
      const int kb = e & 0xFFF;
      const bool row_ok = ((e >> 12) & my_bit) != 0;
      const int valid = (kb == NB - 1) ? (L - kb * BN) : BN;
      for (int j = 0; j < HB; ++j, ++h) {
        const int b = h & 1;
        const int valid_h = valid - j * SN;  // may be <= 0: the whole half is padding
        if (!(ok = warp_wait(&sh->s_full[t][b], (h >> 1) & 1, sh, prm))) break;
        tc_fence_after();
        uint32_t sr[2][32];
        tmem_ld32(tS + b * SN, sr[0]);
        tmem_ld32(tS + b * SN + 32, sr[1]);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i) reg_fence(sr[c][i]);
        // masked halves only: the ragged last key block, or a row half that
        // does not keep this block (blk = 64)
        if (!row_ok || valid_h < SN) {
#pragma unroll
          for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (!row_ok || c * 32 + i >= valid_h) sr[c][i] = __float_as_uint(-INFINITY);
        }
        // raw max (the scale is positive, so it commutes with max), 4 chains
        float mxa = -INFINITY, mxb = -INFINITY, mxc = -INFINITY, mxd = -INFINITY;
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          mxa = max3(mxa, __uint_as_float(sr[0][i]), __uint_as_float(sr[0][i + 1]));
          mxb = max3(mxb, __uint_as_float(sr[0][i + 2]), __uint_as_float(sr[0][i + 3]));
          mxc = max3(mxc, __uint_as_float(sr[1][i]), __uint_as_float(sr[1][i + 1]));
          mxd = max3(mxd, __uint_as_float(sr[1][i + 2]), __uint_as_float(sr[1][i + 3]));
        }
        const float mx = fmaxf(max3(mxa, mxb, mxc), mxd);
        const float m_new = fmaxf(m_ref, mx * sl2);
        const bool resc = m_new > m_ref + kRescaleThreshold;
        float factor = 1.f;
        if (resc) {
          factor = ex2_approx(m_ref - m_new);  // 0 when m_ref is -inf
          l *= factor;
          m_ref = m_new;
        }
        if (h > 0 && __any_sync(0xffffffffu, resc)) {
          // O must be final for half h-1 before it is rescaled (PV_h waits
          // for this half's P, so nothing newer can touch O meanwhile)
          if (!(ok = warp_wait(&sh->pv_done[t][(h - 1) & 1], ((h - 1) >> 1) & 1, sh, prm))) break;
          tc_fence_after();
#pragma unroll
          for (int h2 = 0; h2 < D / 64; ++h2) {
            uint32_t o0[32], o1[32];
            tmem_ld32(tO + h2 * 64, o0);
            tmem_ld32(tO + h2 * 64 + 32, o1);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              reg_fence(o0[i]);
              reg_fence(o1[i]);
              o0[i] = __float_as_uint(__uint_as_float(o0[i]) * factor);
              o1[i] = __float_as_uint(__uint_as_float(o1[i]) * factor);
            }
            tmem_st32(tO + h2 * 64, o0);
            tmem_st32(tO + h2 * 64 + 32, o1);
          }
          tmem_wait_st();
        }
        // p = 2^(s*scale - m): one packed FMA per pair, ex2 on the MUFU unit,
        // packed row sums, bf16 pairs written over the first half of S
        const float mu = (m_ref == -INFINITY) ? 0.f : m_ref;
        const uint64_t scale2 = f2_pack(sl2, sl2);
        const uint64_t negm2 = f2_pack(-mu, -mu);
        uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int col = 2 * i;
          const uint64_t x = f2_fma(f2_pack(__uint_as_float(sr[col >> 5][col & 31]),
                                            __uint_as_float(sr[col >> 5][(col & 31) + 1])),
                                    scale2, negm2);
          float x0, x1;
          f2_unpack(x, x0, x1);
          const float p0 = ex2_approx(x0);
          const float p1 = ex2_approx(x1);
          acc[i & 3] = f2_add(acc[i & 3], f2_pack(p0, p1));
          pk[i] = pack_bf16x2(p0, p1);
        }
        tmem_st32(tS + b * SN, pk);
        {
          float a0, a1, b0, b1;
          f2_unpack(f2_add(acc[0], acc[1]), a0, a1);
          f2_unpack(f2_add(acc[2], acc[3]), b0, b1);
          l += (a0 + a1) + (b0 + b1);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&sh->p_full[t][b]);
      }
      u = next_member(ulist, u + 1, U, tile_mask[t]);
    }
    // ----------------------------------------------------------- epilogue
    bool have_o = ok && ntile[t] > 0;
    if (have_o) {
      have_o = warp_wait(&sh->o_full[t], 0, sh, prm);
      tc_fence_after();
    }
    if (ok) {
      const bool store = grow < L;
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      const float lse_v = l > 0.f ? (m_ref + log2f(l)) * 0.69314718055994531f : -INFINITY;
      const size_t row_elem = (static_cast<size_t>(bh) * L + (store ? grow : 0)) * D;
      const int hh = bh % prm.H;
      const float a = prm.R ? prm.alpha[hh] : 0.f;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t regs[32];
        if (have_o) {
          tmem_ld32(tO + c * 32, regs);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) reg_fence(regs[i]);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) regs[i] = 0u;
        }
        if (store) {
          float v[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(regs[i]) * inv_l;
          if (prm.R) {
            const uint4* rp = reinterpret_cast<const uint4*>(prm.R + row_elem + c * 32);
#pragma unroll
            for (int w = 0; w < 4; ++w) {
              const uint4 rv = __ldg(rp + w);
              const uint32_t rw[4] = {rv.x, rv.y, rv.z, rv.w};
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                v[w * 8 + 2 * i] += a * __uint_as_float(rw[i] << 16);
                v[w * 8 + 2 * i + 1] += a * __uint_as_float(rw[i] & 0xFFFF0000u);
              }
            }
          }
          uint4* op = reinterpret_cast<uint4*>(prm.o + row_elem + c * 32);
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            uint4 ov;
            ov.x = pack_bf16x2(v[w * 8 + 0], v[w * 8 + 1]);
            ov.y = pack_bf16x2(v[w * 8 + 2], v[w * 8 + 3]);
            ov.z = pack_bf16x2(v[w * 8 + 4], v[w * 8 + 5]);
            ov.w = pack_bf16x2(v[w * 8 + 6], v[w * 8 + 7]);
            op[w] = ov;
          }
        }
      }
      if (store) prm.lse[static_cast<size_t>(bh) * L + grow] = lse_v;
    }
  }

  __syncthreads();
  if (warp == 14) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------- host
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// [BH, L, D] bf16 viewed as a 3-D tensor; box = 64 columns x rows x 1.
bool make_map(CUtensorMap* m, const void* base, int D, int L, int BH, int box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(L), static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(L) * D * 2};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int BN>
int run(const bsa_shape& s, const AttnArgs& a, cudaStream_t st) {
  using C = Cfg<D, BN>;
  if (smem_opt_in(reinterpret_cast<const void*>(sparse_attn_kernel<D, BN>), C::SMEM_BYTES) != cudaSuccess)
    return BSA_ECUDA;
  const int BH = s.B * s.H;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, a.q, D, s.L, BH, BM) || !make_map(&mk, a.k, D, s.L, BH, BN) ||
      !make_map(&mv, a.v, D, s.L, BH, BN))
    return BSA_ECUDA;
  Params prm;
  prm.kept_idx = a.kept_idx;
  prm.kept_cnt = a.kept_cnt;
  prm.R = a.R;
  prm.alpha = a.alpha;
  prm.o = a.o;
  prm.lse = a.lse;
  prm.status = a.status;
  prm.H = s.H;
  prm.L = s.L;
  prm.NB = n_blocks(s.L, s.blk);
  prm.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(D)));
  prm.dense = a.kept_idx == nullptr;
  const int n_tiles = (s.L + BM - 1) / BM;
  dim3 grid((n_tiles + 1) / 2, BH);
  sparse_attn_kernel<D, BN><<<grid, kThreads, C::SMEM_BYTES, st>>>(mq, mk, mv, prm);
  return cudaGetLastError() == cudaSuccess ? BSA_OK : BSA_ECUDA;
}

}  // namespace

int launch_sparse_attn_pair(const bsa_shape& s, const AttnArgs& a, cudaStream_t st) {
  if (s.D == 128 && s.blk == 128) return run<128, 128>(s, a, st);
  if (s.D == 128 && s.blk == 64) return run<128, 64>(s, a, st);
  if (s.D == 64 && s.blk == 128) return run<64, 128>(s, a, st);
  if (s.D == 64 && s.blk == 64) return run<64, 64>(s, a, st);
  return BSA_ESHAPE;
}

int launch_sparse_attn(const bsa_shape& s, const AttnArgs& a, cudaStream_t st) {
  if (s.blk == 128) return launch_sparse_attn_tile(s, a, st);
  return launch_sparse_attn_pair(s, a, st);
}

}  // namespace bsa

// Block-sparse attention forward for sm_100a, 128-token key blocks:
// persistent, one 128-row query tile at a time per CTA (one CTA per SM).
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
// Schedule.  Work item w = (b*H + h) * NT + query block.  CTAs take items
// from one atomic counter, in order, so the items in flight at any time are
// neighbouring query blocks of the same head (its K/V stays in L2) and uneven
// kept lists do not unbalance the SMs.  The TMA-Q/K warp fetches the next item
// and passes it to the other roles through a 4-deep queue in shared memory.
// The counter lives in a slot of a small in-library ring (one slot per launch,
// round robin); the last CTA of a launch resets its slot, so each launch finds
// its slot at zero as long as fewer than kSchedSlots launches overlap.
//
// Tensor memory (512 columns): S0 | S1 | S2 | O at D = 128 (S0 | S1 | S2 |
// O0 | O1 at D = 64).  S is triple buffered, so the tensor core can compute S
// for blocks n+1 and n+2 while the softmax works on block n, and the S of
// block n+3 waits only for the PV of block n.  P of block n (bf16 pairs)
// overwrites the first 64 columns of its S buffer.  With one O buffer the
// first PV of an item waits until the epilogue has read the previous item's
// O out; the S MMAs and the softmax of the new item's first blocks run
// meanwhile.  All MMAs are M=128, N=128 (or N=D), K=16: full-rate shapes.
//
// Warp roles (16 warps):
//   warp 0       item queue; TMA: Q of every item (kQBuffers buffers), K ring
//   warp 1       TMA: V ring; TMEM allocation
//   warp 2       S issuer:  S_n = Q K_n^T into S[n%3] (S[n%2] when fused)
//   warp 3       PV issuer: O[item%OB] += P_n V_n, P read from TMEM (OB = 1
//                at D = 128, 2 at D = 64)
//   warps 4-7    softmax of rows 32q+0..15 of every TMEM quarter q
//   warps 8-11   softmax of rows 32q+16..31
//   warps 12-15  epilogue: O/l (+ alpha*R) -> bf16, LSE
// The softmax reads S with 16-lane TMEM loads: a thread holds two rows and,
// per 8-key chunk, one adjacent key pair of each, which is exactly the bf16
// pair of one P column; 4 threads share a row and combine maxima and sums with
// two shuffles.  The two softmax warpgroups own disjoint rows and never wait
// for each other, so one can exponentiate while the other loads.
//
// FP8 Q.K^T (kF8, D = 128): the Q and K tiles are E4M3 codes (128-byte
// swizzled rows of 128 codes), S = Q K^T runs as kind::f8f6f4 MMAs (32 codes of
// K per instruction), and the softmax scales a block's logits by s_q * s_k,
// the dequantization scales of the query and key blocks (the key block's scale
// is loaded one block ahead).  V, P and O are as in the bf16 path.
//
// Row gathers (kGather, D = 128): token t of the attention's order is row
// in_rows[t] of the grid-order Q, K and V; each 128-row tile arrives as 64
// four-row TMA gathers (2 per lane of the producer warp), and the epilogue
// writes O, LSE and reads R through the same rows.
//
// Online softmax in the log2 domain in fp32.  The reference max is only
// raised when a block max exceeds it by more than 8 (so P <= 2^8); O is then
// rescaled in TMEM (after the previous PV completed), and the final 1/l uses
// the same reference.
//
// Fused refresh (kFused).  Every key block is visited once; the PV of a kept
// block accumulates into OK, that of any other block into OR (TMEM at D = 128:
// S0 | S1 | OK | OR, so S is double buffered and O single buffered across
// items, and the PV of an item waits until the epilogue has read the previous
// item's O).  One shared reference
// max serves both; the softmax keeps the total row sum and the kept row sum.
// The epilogue writes the dense output (OK + OR) / l, the sparse output
// OK / l_kept, both LSEs, R = bf16(bf16(O_dense) - bf16(O_sparse)) and the kept
// share of the attention weight l_kept / l (RECAP section 1 and section 3.4
// with Fig. 3: a dense refresh renews the refinement; GSRS abstract: exact
// attention weights within the attention computation).  Membership of a block
// in the kept set comes from the ascending kept list; entries that are out of
// range or out of order are skipped and flagged.
//
// Every wait is bounded (2 s of globaltimer); a timeout sets BSA_DEV_TIMEOUT
// in the caller's status word and makes every role give up; the MMA issuers
// and TMA producers wait (bounded) for their operations in flight before TMEM
// is released.
#include <cuda.h>
#include <cuda_bf16.h>

#include <atomic>
#include <cmath>

#include "internal.cuh"
#include "sm100.cuh"

namespace bsa {
namespace tile_attn {

using namespace sm100;

constexpr int kThreads = 512;
constexpr int BM = 128;                         // query rows per work item
constexpr int BN = 128;                         // keys per block
constexpr uint64_t kTimeoutNs = 2000000000ull;  // 2 s
constexpr float kRescaleThreshold = 8.0f;       // log2 units
// Key pairs whose exponentials are evaluated on the FMA pipe by exp2_poly
// instead of the exp unit: bit 2k is row rA's pair in 8-key chunk k of the 16 a
// softmax thread handles per block, bit 2k+1 row rA+8's
constexpr uint32_t kPolyPairs = 0x0000C000u;
// Q tiles in shared memory across items: one leaves room for a third K slot
constexpr int kQBuffers = 1;
constexpr int kQueue = 4;                       // item queue depth
constexpr int kItemReaders = 32 * 3 + 256 + 128;  // threads of the roles that read the queue
// registers per thread: launch 65536 / 512 = 128, then re-balanced per warpgroup
constexpr int kRegsCtl = 56;        // TMA producers, MMA issuers
constexpr int kRegsSoftmax = 168;   // two warpgroups
constexpr int kRegsEpilogue = 120;
static_assert(128 * kRegsCtl + 256 * kRegsSoftmax + 128 * kRegsEpilogue <= 512 * 128, "register split exceeds launch");

// Work counters.  Each launch draws its work items from one slot of a ring,
// the host assigning slots round robin, one per launch.  A slot is owned by
// one launch from its first CTA to its last: the state word holds the owner's
// tag (from %gridid, so two replays of one captured graph differ), how many of
// its CTAs joined and how many have left.  The last CTA to leave returns the
// counter to zero and frees the slot, so a launch needs no memset and the call
// allocates nothing.  A CTA that finds its slot owned by another launch (more
// than kSchedSlots launches executing at once, or one captured graph replayed
// on two streams at the same time) does no work and flags
// BSA_DEV_SCHED_CONFLICT; the slot stays consistent for later launches.
constexpr int kSchedSlots = 256;
struct SchedSlot {
  unsigned long long state;  // tag << 32 | joined << 16 | left; 0 = free
  unsigned int next;         // next work item; 0 whenever the slot is free
  unsigned int last_tag;     // tag of the last launch that freed the slot
  unsigned int pad[28];
};
__device__ SchedSlot g_sched[kSchedSlots];
constexpr int kCasTries = 1 << 16;

struct Params {
  const int32_t* kept_idx;
  const int32_t* kept_cnt;
  const __nv_bfloat16* R;
  const float* alpha;
  __nv_bfloat16* o;
  float* lse;
  __nv_bfloat16* o2;     // fused refresh: sparse output
  float* lse2;           //                sparse LSE
  __nv_bfloat16* r_out;  //                refinement (nullable)
  float* mass;           //                kept attention share (nullable)
  const int32_t* out_rows;  // output row map (nullable = identity)
  int32_t* status;
  const float* q_scale;  // FP8 Q.K^T: dequantization scale per (b, h, block) of Q and of K
  const float* k_scale;
  const int32_t* in_rows;  // row gathers: token t is row in_rows[t] of q, k, v
  int H, L, NB, NT, n_work;
  int n_rows;              // B * H * L: the first row past q, k, v (reads zeros)
  float scale_log2;
  int dense;
  int sched_slot;
  // interval mode: the kept blocks as pairs [B,H,NB,W,2] and pairs per row [B,H,NB]
  const int32_t* intervals;
  const int32_t* n_int;
  int W;
};

// kF8: Q and K are E4M3 (one byte per element), S = Q.K^T runs as a
// kind::f8f6f4 MMA; V, P and O stay bf16.
template <int D, bool kF8>
struct Cfg {
  static constexpr int QK_ELEM = kF8 ? 1 : 2;        // bytes per Q / K element
  static constexpr int Q_BYTES = BM * D * QK_ELEM;
  static constexpr int NQ = kQBuffers;            // Q buffers across items
  static constexpr int K_BYTES = BN * D * QK_ELEM;
  static constexpr int V_BYTES = BN * D * 2;
  static constexpr int STATS_BYTES = 2 * 3 * BM * 4;  // [item parity][l, m, l_kept][row]
  static constexpr int MISC_BYTES = 512;
  static constexpr int AVAIL = 227 * 1024 - 1024 - NQ * Q_BYTES - STATS_BYTES - MISC_BYTES;
  static constexpr int SLOTS = AVAIL / V_BYTES;   // equal K and V slots (bf16)
  static constexpr int NSK = kF8 ? 4 : (((SLOTS + 1) / 2) > 4 ? 4 : (SLOTS + 1) / 2);
  static constexpr int NSV_FIT = kF8 ? (AVAIL - NSK * K_BYTES) / V_BYTES : SLOTS / 2;
  static constexpr int NSV = NSV_FIT > 4 ? 4 : NSV_FIT;
  static_assert(NSK >= 2 && NSV >= 2, "shared memory too small for double-buffered K and V");
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = NQ * Q_BYTES;
  static constexpr int OFF_V = OFF_K + NSK * K_BYTES;
  static constexpr int OFF_STATS = OFF_V + NSV * V_BYTES;
  static constexpr int OFF_MISC = OFF_STATS + STATS_BYTES;
  static constexpr int SMEM_BYTES = OFF_MISC + MISC_BYTES + 1024;
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
  static constexpr int COL_S = 0;        // S[b] at b*BN
  // 128-byte rows of the swizzled tiles: Q/K panels of 64 bf16 or 128 E4M3
  static constexpr int QK_PANEL_ELEMS = 128 / QK_ELEM;
  static constexpr int QK_PANELS = D / QK_PANEL_ELEMS;
  static constexpr int PANELS = D / 64;              // V panels
  static constexpr int S_KSTEPS = D * QK_ELEM / 32;  // 32 bytes of K per MMA
};

struct Shared {
  uint64_t full_k[4], empty_k[4], full_v[4], empty_v[4];
  uint64_t q_full[2], q_empty[2];
  uint64_t s_full[3], p_full[3], pv_done[3];
  uint64_t o_full[2], o_empty[2];
  uint64_t stats_full[2], stats_free[2];
  uint64_t drain[2];
  uint64_t item_full[kQueue], item_empty[kQueue];
  int items[kQueue];
  uint32_t tmem_base;
  volatile int abort_flag;
  int joined;  // this CTA fetches work from its scheduler slot
};
static_assert(sizeof(Shared) <= 512, "misc region too small");

__device__ __forceinline__ void flag_status(const Params& prm, int bits) {
  if (prm.status) atomicOr(prm.status, bits);
}

__device__ __forceinline__ uint32_t launch_tag() {
  uint64_t g;
  asm volatile("mov.u64 %0, %%gridid;" : "=l"(g));
  return (static_cast<uint32_t>(g) << 1) | 1u;  // never 0 (0 marks a free slot)
}

// Joins this CTA to its launch's use of the slot; false: fetch no work (the
// slot belongs to another launch, or this launch has already finished).
__device__ bool sched_join(SchedSlot* s, uint32_t tag, const Params& prm) {
  unsigned long long cur = atomicAdd(&s->state, 0ull);
  for (int t = 0; t < kCasTries; ++t) {
    const uint32_t owner = static_cast<uint32_t>(cur >> 32);
    const uint32_t joined = static_cast<uint32_t>(cur >> 16) & 0xffffu, left = static_cast<uint32_t>(cur) & 0xffffu;
    unsigned long long want;
    if (owner == 0) {
      if (atomicAdd(&s->last_tag, 0u) == tag) return false;  // this launch already finished
      want = (static_cast<unsigned long long>(tag) << 32) | (1ull << 16);
    } else if (owner == tag) {
      if (joined != 0 && left == joined) return false;  // finishing: nothing left to fetch
      want = cur + (1ull << 16);
    } else {
      flag_status(prm, BSA_DEV_SCHED_CONFLICT);
      return false;
    }
    const unsigned long long got = atomicCAS(&s->state, cur, want);
    if (got == cur) {
      __threadfence();
      return true;
    }
    cur = got;
  }
  flag_status(prm, BSA_DEV_SCHED_CONFLICT);
  return false;
}

// Leaves the slot after this CTA's last fetch; the last CTA to leave resets
// the counter and frees the slot.
__device__ void sched_leave(SchedSlot* s, uint32_t tag, const Params& prm) {
  __threadfence();
  unsigned long long cur = atomicAdd(&s->state, 0ull);
  for (int t = 0; t < kCasTries; ++t) {
    const unsigned long long want = cur + 1ull;
    const unsigned long long got = atomicCAS(&s->state, cur, want);
    if (got == cur) {
      if ((static_cast<uint32_t>(want >> 16) & 0xffffu) == (static_cast<uint32_t>(want) & 0xffffu)) {
        atomicExch(&s->next, 0u);
        atomicExch(&s->last_tag, tag);
        __threadfence();
        atomicExch(&s->state, 0ull);
      }
      return;
    }
    cur = got;
  }
  flag_status(prm, BSA_DEV_SCHED_CONFLICT);
}

// 2^x for a pair of floats (x <= 127) on the FMA and integer pipes, without
// the exp unit: x = j + f with j the nearest integer and f in [-1/2, 1/2]
// (adding 1.5 * 2^23 rounds x to an integer, whose value lands in the low
// mantissa bits); 2^f by a degree-3 polynomial fitted to a relative error of
// 7.5e-5 on that interval, far below the bf16 rounding of P; 2^j added to the
// exponent field.  x below -125 gives 2^-125 (about 2e-38) instead of ~0.
__device__ __forceinline__ uint64_t exp2_poly(uint64_t x) {
  float x0, x1;
  f2_unpack(x, x0, x1);
  x0 = fmaxf(x0, -125.f);
  x1 = fmaxf(x1, -125.f);
  const uint64_t xc = f2_pack(x0, x1);
  const uint64_t t = f2_add(xc, f2_pack(12582912.f, 12582912.f));
  const uint64_t j = f2_add(t, f2_pack(-12582912.f, -12582912.f));
  const uint64_t fr = f2_fma(j, f2_pack(-1.f, -1.f), xc);
  uint64_t p = f2_fma(f2_pack(0.055171772837638855f, 0.055171772837638855f), fr,
                      f2_pack(0.24261115491390228f, 0.24261115491390228f));
  p = f2_fma(p, fr, f2_pack(0.6932609677314758f, 0.6932609677314758f));
  p = f2_fma(p, fr, f2_pack(0.9999280571937561f, 0.9999280571937561f));
  float p0, p1, t0, t1;
  f2_unpack(p, p0, p1);
  f2_unpack(t, t0, t1);
  return f2_pack(__uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23)),
                 __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23)));
}

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

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, Shared* sh, const Params& prm) {
  const bool ok = wait_bounded(bar, parity, sh, prm);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try(bar, parity) && globaltimer_ns() - t0 < kTimeoutNs) {
  }
}

// Next work item of this CTA (queue position i), or -1 at the end / on abort.
// Every reading thread releases its queue slot right after reading it.
__device__ __forceinline__ int next_item(int i, Shared* sh, const Params& prm) {
  const int qs = i % kQueue;
  if (!warp_wait(&sh->item_full[qs], (i / kQueue) & 1, sh, prm)) return -1;
  const int w = sh->items[qs];
  mbar_arrive(&sh->item_empty[qs]);
  return w;
}

// One work item: a 128-row query block of one (batch, head) and its key list.
struct Item {
  int bh, qb, cnt;
  const int32_t* list;   // null in dense mode
  bool bad_cnt;          // the count was outside [0, NB] and was clamped (interval mode: malformed pairs)
  const int32_t* klist;  // fused refresh: the kept list (ascending) ...
  int kcnt;              // ... and its length
};

template <bool kFused>
__device__ __forceinline__ Item item_of(int w, const Params& prm) {
  Item it;
  it.bh = w / prm.NT;
  it.qb = w - it.bh * prm.NT;
  it.bad_cnt = false;
  it.klist = nullptr;
  it.kcnt = 0;
  if (kFused) {
    const size_t r = static_cast<size_t>(it.bh) * prm.NB + it.qb;
    const int c = __ldg(prm.kept_cnt + r);
    it.bad_cnt = c < 0 || c > prm.NB;
    it.kcnt = c < 0 ? 0 : (c > prm.NB ? prm.NB : c);
    it.klist = prm.kept_idx + r * prm.NB;
    it.cnt = prm.NB;
    it.list = nullptr;
  } else if (prm.dense) {
    it.cnt = prm.NB;
    it.list = nullptr;
  } else {
    const size_t r = static_cast<size_t>(it.bh) * prm.NB + it.qb;
    const int c = __ldg(prm.kept_cnt + r);
    it.bad_cnt = c < 0 || c > prm.NB;
    it.cnt = c < 0 ? 0 : (c > prm.NB ? prm.NB : c);
    it.list = prm.kept_idx + r * prm.NB;
  }
  return it;
}

// Key block of entry n, or -1 for an out-of-range entry (skipped by every role).
__device__ __forceinline__ int entry_kb(const Item& it, int n, int NB) {
  const int kb = it.list ? __ldg(it.list + n) : n;
  return static_cast<unsigned>(kb) < static_cast<unsigned>(NB) ? kb : -1;
}

// Interval mode (CalibAtt appendix, Fig. S10: the kernel walks the skip
// lists): the item carries its row's (start, end) pairs, checked as the decode
// checks them (ascending, within [0, NB], non-empty; a malformed row is empty
// and flagged), and every role walks them in order with its own cursor.
struct ItemIv : Item {
  const int32_t* pairs;
};
struct Walk {
  int p = -1, kb = 0, end = 0;
};

__device__ __forceinline__ ItemIv item_iv_of(int w, const Params& prm) {
  ItemIv it;
  it.bh = w / prm.NT;
  it.qb = w - it.bh * prm.NT;
  it.klist = nullptr;
  it.kcnt = 0;
  it.list = nullptr;
  const size_t r = static_cast<size_t>(it.bh) * prm.NB + it.qb;
  const int ni = __ldg(prm.n_int + r);
  it.pairs = prm.intervals + r * prm.W * 2;
  bool bad = ni < 0 || ni > prm.W;
  int cnt = 0, prev = 0;
  for (int p = 0; !bad && p < ni; ++p) {
    const int a = __ldg(it.pairs + 2 * p), b = __ldg(it.pairs + 2 * p + 1);
    bad = a < prev || a >= b || b > prm.NB;
    cnt += b - a;
    prev = b;
  }
  it.bad_cnt = bad;
  it.cnt = bad ? 0 : cnt;
  return it;
}

// The next key block of a validated row (entries visited in order).
__device__ __forceinline__ int entry_kb(const ItemIv& it, int, int, Walk& w) {
  while (w.kb >= w.end) {
    ++w.p;
    w.kb = __ldg(it.pairs + 2 * w.p);
    w.end = __ldg(it.pairs + 2 * w.p + 1);
  }
  return w.kb++;
}

template <bool kFused, bool kIntervals>
__device__ __forceinline__ auto item_at(int w, const Params& prm) {
  if constexpr (kIntervals)
    return item_iv_of(w, prm);
  else
    return item_of<kFused>(w, prm);
}

// Key block of entry n in either mode (the cursor is used by interval mode only).
template <bool kIntervals, class It>
__device__ __forceinline__ int next_kb(const It& it, int n, int NB, Walk& w) {
  if constexpr (kIntervals)
    return entry_kb(it, n, NB, w);
  else
    return entry_kb(it, n, NB);
}

// Fused refresh: is key block j (visited in ascending order) in the kept list?
// kp walks the list; entries below j were out of order or repeated.
__device__ __forceinline__ bool kept_at(const Item& it, int j, int& kp, bool& bad) {
  int e = kp < it.kcnt ? __ldg(it.klist + kp) : INT_MAX;
  while (e < j) {
    bad = true;
    ++kp;
    e = kp < it.kcnt ? __ldg(it.klist + kp) : INT_MAX;
  }
  if (e == j) {
    ++kp;
    return true;
  }
  return false;
}

// Row gathers: the 128 tokens t0..t0+127 of the attention's order, rows
// in_rows[t] of (b, h) = it.bh, as two 64-column panels of a 128-row tile at
// dst (the layout a tiled load gives).  Lane l fetches tokens 4l..4l+3 with one
// 4-row gather per panel; tokens past L and rows outside [0, L) read zeros
// (the latter also flagged).  The caller has set the barrier's byte count.
__device__ __forceinline__ void gather_tile(uint8_t* dst, const CUtensorMap* map, uint64_t* bar, int bh, int t0,
                                            int lane, const Params& prm) {
  const int t = t0 + 4 * lane;
  int g[4];
  if (t + 4 <= prm.L) {
    const int4 v = __ldg(reinterpret_cast<const int4*>(prm.in_rows + t));
    g[0] = v.x, g[1] = v.y, g[2] = v.z, g[3] = v.w;
  } else {
#pragma unroll
    for (int e = 0; e < 4; ++e) g[e] = t + e < prm.L ? __ldg(prm.in_rows + t + e) : -1;
  }
  bool bad = false;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const bool in = static_cast<unsigned>(g[e]) < static_cast<unsigned>(prm.L);
    bad |= !in && t + e < prm.L;
    g[e] = in ? bh * prm.L + g[e] : prm.n_rows;
  }
  if (bad) flag_status(prm, BSA_DEV_BAD_INDEX);
#pragma unroll
  for (int pnl = 0; pnl < 2; ++pnl)
    tma_gather4(dst + pnl * (BM * 128) + lane * 512, map, bar, pnl * 64, g[0], g[1], g[2], g[3]);
}

template <int D, bool kFused, bool kF8, bool kGather, bool kIntervals>
__global__ void __launch_bounds__(kThreads, 1)
    sparse_attn_tile_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                            const __grid_constant__ CUtensorMap tmV, const Params prm) {
  using C = Cfg<D, kF8>;
  static_assert(!kGather || (D == 128 && !kFused && !kF8), "row gathers: bf16, D = 128, not the fused refresh");
  static_assert(!kIntervals || (!kFused && !kF8 && !kGather), "interval pairs: bf16, not the fused refresh");
  // TMEM (512 columns): NS buffers of S (128 columns each) then OB buffers of
  // the accumulator(s) of an item (D columns each; the fused refresh keeps two
  // per item, OK and OR).  D = 128: S0|S1|S2|O, fused S0|S1|OK|OR.
  constexpr int OB_RESCALE = kFused ? 2 : 1;  // accumulators per item
  constexpr int NS = kFused ? (512 - 2 * D) / BN : 3;
  constexpr int OB_FIT = (512 - NS * BN) / (OB_RESCALE * D);
  constexpr int OB = OB_FIT > 2 ? 2 : OB_FIT;  // O buffers across items
  constexpr int COL_O = NS * BN;
  static_assert(NS >= 2 && NS <= 3 && OB >= 1, "TMEM layout");
  constexpr int NSK = C::NSK;
  constexpr int NSV = C::NSV;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Shared* sh = reinterpret_cast<Shared*>(smem + C::OFF_MISC);
  float* stats = reinterpret_cast<float*>(smem + C::OFF_STATS);
  uint8_t* q_smem = smem + C::OFF_Q;
  uint8_t* k_ring = smem + C::OFF_K;
  uint8_t* v_ring = smem + C::OFF_V;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int NB = prm.NB;
  const int L = prm.L;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 4; ++s) {
      mbar_init(&sh->full_k[s], 1);
      mbar_init(&sh->empty_k[s], 1);
      mbar_init(&sh->full_v[s], 1);
      mbar_init(&sh->empty_v[s], 1);
      mbar_init(&sh->item_full[s], 1);
      mbar_init(&sh->item_empty[s], kItemReaders);
    }
    for (int j = 0; j < 3; ++j) {
      mbar_init(&sh->s_full[j], 1);
      mbar_init(&sh->p_full[j], 256);
      mbar_init(&sh->pv_done[j], 1);
    }
    for (int j = 0; j < 2; ++j) {
      mbar_init(&sh->q_full[j], 1);
      mbar_init(&sh->q_empty[j], 1);
      mbar_init(&sh->o_full[j], 1);
      mbar_init(&sh->o_empty[j], 128);
      mbar_init(&sh->stats_full[j], 256);
      mbar_init(&sh->stats_free[j], 128);
      mbar_init(&sh->drain[j], 1);
    }
    sh->abort_flag = 0;
    sh->joined = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(&sh->tmem_base, 512);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;

  if (warp < 4) {
    setmaxnreg_dec<kRegsCtl>();
    if (warp == 0) {
      // ---------------------------------- item queue, TMA: Q and the K ring
      SchedSlot* sched = &g_sched[prm.sched_slot];
      const uint32_t tag = launch_tag();
      int joined = 0;
      if (lane == 0) {
        joined = sched_join(sched, tag, prm) ? 1 : 0;
        sh->joined = joined;
      }
      joined = __shfl_sync(0xffffffffu, joined, 0);
      int u = 0;
      bool ok = true;
      for (int i = 0;; ++i) {
        const int qs = i % kQueue;
        if (i >= kQueue && !(ok = warp_wait(&sh->item_empty[qs], ((i / kQueue) - 1) & 1, sh, prm))) break;
        int w = 0;
        if (lane == 0) {
          w = joined ? static_cast<int>(atomicAdd(&sched->next, 1u)) : -1;
          if (w >= prm.n_work) w = -1;
          sh->items[qs] = w;
          mbar_arrive(&sh->item_full[qs]);
        }
        w = __shfl_sync(0xffffffffu, w, 0);
        if (w < 0) break;
        const auto it = item_at<kFused, kIntervals>(w, prm);
        if (it.bad_cnt && lane == 0) flag_status(prm, BSA_DEV_BAD_INDEX);
        const int qb = i % C::NQ;
        if (i >= C::NQ && !(ok = warp_wait(&sh->q_empty[qb], ((i - C::NQ) / C::NQ) & 1, sh, prm))) break;
        if constexpr (kGather) {
          if (lane == 0) mbar_arrive_expect_tx(&sh->q_full[qb], C::Q_BYTES);
          __syncwarp();
          gather_tile(q_smem + qb * C::Q_BYTES, &tmQ, &sh->q_full[qb], it.bh, it.qb * BM, lane, prm);
        } else if (lane == 0) {
          mbar_arrive_expect_tx(&sh->q_full[qb], C::Q_BYTES);
          for (int pnl = 0; pnl < C::QK_PANELS; ++pnl)
            tma_load_3d(q_smem + qb * C::Q_BYTES + pnl * BM * 128, &tmQ, &sh->q_full[qb], pnl * C::QK_PANEL_ELEMS,
                        it.qb * BM,
                        it.bh);
        }
        __syncwarp();
        Walk wk;
        for (int n = 0; ok && n < it.cnt; ++n) {
          const int kb = next_kb<kIntervals>(it, n, NB, wk);
          if (kb < 0) {
            if (lane == 0) flag_status(prm, BSA_DEV_BAD_INDEX);
            continue;
          }
          const int slot = u % NSK;
          if (u >= NSK && !(ok = warp_wait(&sh->empty_k[slot], ((u / NSK) - 1) & 1, sh, prm))) break;
          if constexpr (kGather) {
            if (lane == 0) mbar_arrive_expect_tx(&sh->full_k[slot], C::K_BYTES);
            __syncwarp();
            gather_tile(k_ring + slot * C::K_BYTES, &tmK, &sh->full_k[slot], it.bh, kb * BN, lane, prm);
          } else if (lane == 0) {
            mbar_arrive_expect_tx(&sh->full_k[slot], C::K_BYTES);
            for (int pnl = 0; pnl < C::QK_PANELS; ++pnl)
              tma_load_3d(k_ring + slot * C::K_BYTES + pnl * BN * 128, &tmK, &sh->full_k[slot],
                          pnl * C::QK_PANEL_ELEMS, kb * BN,
                          it.bh);
          }
          __syncwarp();
          ++u;
        }
        if (!ok) break;
      }
      if (!ok && lane == 0) {
        for (int v = u - NSK < 0 ? 0 : u - NSK; v < u; ++v) drain_wait(&sh->full_k[v % NSK], (v / NSK) & 1);
      }
      __syncwarp();
    } else if (warp == 1) {
      // ------------------------------------------------------ TMA: V ring
      int u = 0;
      bool ok = true;
      for (int i = 0; ok; ++i) {
        const int w = next_item(i, sh, prm);
        if (w < 0) break;
        const auto it = item_at<kFused, kIntervals>(w, prm);
        Walk wk;
        for (int n = 0; n < it.cnt; ++n) {
          const int kb = next_kb<kIntervals>(it, n, NB, wk);
          if (kb < 0) continue;
          const int slot = u % NSV;
          if (u >= NSV && !(ok = warp_wait(&sh->empty_v[slot], ((u / NSV) - 1) & 1, sh, prm))) break;
          if constexpr (kGather) {
            if (lane == 0) mbar_arrive_expect_tx(&sh->full_v[slot], C::V_BYTES);
            __syncwarp();
            gather_tile(v_ring + slot * C::V_BYTES, &tmV, &sh->full_v[slot], it.bh, kb * BN, lane, prm);
          } else if (lane == 0) {
            mbar_arrive_expect_tx(&sh->full_v[slot], C::V_BYTES);
            for (int pnl = 0; pnl < C::PANELS; ++pnl)
              tma_load_3d(v_ring + slot * C::V_BYTES + pnl * BN * 128, &tmV, &sh->full_v[slot], pnl * 64, kb * BN,
                          it.bh);
          }
          __syncwarp();
          ++u;
        }
      }
      if (!ok && lane == 0)
        for (int v = u - NSV < 0 ? 0 : u - NSV; v < u; ++v) drain_wait(&sh->full_v[v % NSV], (v / NSV) & 1);
      __syncwarp();
    } else if (warp == 2) {
      // ---------------------------------------------------------- S issuer
      constexpr uint32_t idS = kF8 ? idesc_e4m3_f32(BM, BN) : idesc_bf16_f32(BM, BN, false, false);
      const uint32_t q_base = smem_u32(q_smem);
      const uint32_t k_base = smem_u32(k_ring);
      int u = 0;
      bool ok = true;
      for (int i = 0; ok; ++i) {
        const int w = next_item(i, sh, prm);
        if (w < 0) break;
        const auto it = item_at<kFused, kIntervals>(w, prm);
        const int qb = i % C::NQ;
        if (!(ok = warp_wait(&sh->q_full[qb], (i / C::NQ) & 1, sh, prm))) break;
        const uint32_t qa = q_base + qb * C::Q_BYTES;
        Walk wk;
        for (int n = 0; n < it.cnt; ++n) {
          if (next_kb<kIntervals>(it, n, NB, wk) < 0) continue;
          const int sk = u % NSK;
          const int b = u % NS;
          if (!(ok = warp_wait(&sh->full_k[sk], (u / NSK) & 1, sh, prm))) break;
          // S[b] held P of block u - NS: its PV must have read it
          if (u >= NS && !(ok = warp_wait(&sh->pv_done[b], ((u - NS) / NS) & 1, sh, prm))) break;
          tc_fence_after();
          if (lane == 0) {
            const uint32_t ka = k_base + sk * C::K_BYTES;
#pragma unroll
            for (int kk = 0; kk < C::S_KSTEPS; ++kk) {
              const uint32_t off_q = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
              const uint32_t off_k = (kk >> 2) * (BN * 128) + (kk & 3) * 32;
              if constexpr (kF8)
                mma_ss_f8(tmem + C::COL_S + b * BN, sdesc_sw128(qa + off_q, 16, 1024),
                          sdesc_sw128(ka + off_k, 16, 1024), idS, kk > 0 ? 1u : 0u);
              else
                mma_ss(tmem + C::COL_S + b * BN, sdesc_sw128(qa + off_q, 16, 1024),
                       sdesc_sw128(ka + off_k, 16, 1024), idS, kk > 0 ? 1u : 0u);
            }
            tc_commit(&sh->s_full[b]);
            tc_commit(&sh->empty_k[sk]);
          }
          __syncwarp();
          ++u;
        }
        if (!ok) break;
        if (lane == 0) tc_commit(&sh->q_empty[qb]);
        __syncwarp();
      }
      if (!ok && lane == 0) {
        tc_commit(&sh->drain[0]);
        drain_wait(&sh->drain[0], 0);
      }
      __syncwarp();
    } else {
      // --------------------------------------------------------- PV issuer
      constexpr uint32_t idPV = idesc_bf16_f32(BM, D, false, true);
      const uint32_t v_base = smem_u32(v_ring);
      int u = 0;
      bool ok = true;
      for (int i = 0; ok; ++i) {
        const int w = next_item(i, sh, prm);
        if (w < 0) break;
        const auto it = item_at<kFused, kIntervals>(w, prm);
        const int ob = i % OB;
        if (i >= OB && !(ok = warp_wait(&sh->o_empty[ob], ((i - OB) / OB) & 1, sh, prm))) break;
        bool first = true, first_rest = true;
        int kp = 0;
        bool bad = false;
        Walk wk;
        for (int n = 0; n < it.cnt; ++n) {
          const int kb = next_kb<kIntervals>(it, n, NB, wk);
          if (kb < 0) continue;
          const bool kept = !kFused || kept_at(it, kb, kp, bad);
          const int sv = u % NSV;
          const int b = u % NS;
          if (!(ok = warp_wait(&sh->p_full[b], (u / NS) & 1, sh, prm))) break;
          if (!(ok = warp_wait(&sh->full_v[sv], (u / NSV) & 1, sh, prm))) break;
          tc_fence_after();
          const bool fresh = kept ? first : first_rest;
          if (lane == 0) {
            const uint32_t va = v_base + sv * C::V_BYTES;
            const uint32_t dst = tmem + COL_O + (kFused ? (kept ? 0 : D) : ob * D);
#pragma unroll
            for (int kk = 0; kk < BN / 16; ++kk)
              mma_ts(dst, tmem + C::COL_S + b * BN + kk * 8, sdesc_sw128(va + kk * 2048, BN * 128, 1024), idPV,
                     (!fresh || kk > 0) ? 1u : 0u);
            tc_commit(&sh->pv_done[b]);
            tc_commit(&sh->empty_v[sv]);
          }
          __syncwarp();
          if (kept)
            first = false;
          else
            first_rest = false;
          ++u;
        }
        if (!ok) break;
        if (kFused && (bad || kp < it.kcnt) && lane == 0) flag_status(prm, BSA_DEV_BAD_INDEX);
        if (lane == 0) tc_commit(&sh->o_full[ob]);
        __syncwarp();
      }
      if (!ok && lane == 0) {
        tc_commit(&sh->drain[1]);
        drain_wait(&sh->drain[1], 0);
      }
      __syncwarp();
    }
  } else if (warp < 12) {
    // ------------------------------------------------------------- softmax
    setmaxnreg_inc<kRegsSoftmax>();
    const int grp = (warp - 4) >> 2;     // 0: rows 32q+0..15, 1: rows 32q+16..31
    const int quarter = warp & 3;
    const int j4 = lane & 3;             // column slot within each chunk
    const int rA = quarter * 32 + grp * 16 + (lane >> 2);  // the thread's two rows: rA, rA + 8
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32 + grp * 16) << 16;
    const float sl2_base = prm.scale_log2;
    int u = 0;
    bool ok = true;
    for (int i = 0; ok; ++i) {
      const int w = next_item(i, sh, prm);
      if (w < 0) break;
      const auto it = item_at<kFused, kIntervals>(w, prm);
      const int ob = i % OB;
      const int sb = i & 1;  // statistics buffer
      const uint32_t tO = tmem + lane_off + COL_O + ob * D;
      // FP8: the logits of block pair (i, j) carry the scales of Q block i and K block j
      const float sl2_item =
          kF8 ? sl2_base * __ldg(prm.q_scale + static_cast<size_t>(it.bh) * prm.NB + it.qb) : sl2_base;
      float mA = -INFINITY, mB = -INFINITY;  // reference max of rows rA, rA+8 (log2 units)
      float lA = 0.f, lB = 0.f;              // this thread's share of the row sums
      float kA = 0.f, kB = 0.f;              // fused refresh: the same over the kept blocks
      int nt = 0;
      int kp = 0;
      bool bad = false;
      // FP8: the K block scale of list entry n, loaded one block ahead
      const float* ks_row = kF8 ? prm.k_scale + static_cast<size_t>(it.bh) * prm.NB : nullptr;
      auto k_scale_at = [&](int n) {  // list mode only (the FP8 path takes no intervals)
        const int kb = entry_kb(static_cast<const Item&>(it), n, NB);
        return kb >= 0 ? __ldg(ks_row + kb) : 1.f;
      };
      float ks_next = kF8 && it.cnt > 0 ? k_scale_at(0) : 1.f;
      Walk wk;
      for (int n = 0; n < it.cnt; ++n) {
        const int kb = next_kb<kIntervals>(it, n, NB, wk);
        float ks = 1.f;
        if constexpr (kF8) {
          ks = ks_next;
          if (n + 1 < it.cnt) ks_next = k_scale_at(n + 1);
        }
        if (kb < 0) continue;
        const bool kept = !kFused || kept_at(it, kb, kp, bad);
        const int b = u % NS;
        const uint32_t tS = tmem + lane_off + C::COL_S + b * BN;
        const float sl2 = kF8 ? sl2_item * ks : sl2_item;
        const uint64_t scale2 = f2_pack(sl2, sl2);
        if (!(ok = warp_wait(&sh->s_full[b], (u / NS) & 1, sh, prm))) break;
        tc_fence_after();
        // s[chunk][0..1]: row rA, keys 8*chunk + 2*j4 + {0,1}; s[chunk][2..3]: row rA+8
        uint32_t sr[2][32];
        tmem_ld_16x256b_x8(tS, sr[0]);
        tmem_ld_16x256b_x8(tS + 64, sr[1]);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 2; ++q)
#pragma unroll
          for (int e = 0; e < 32; ++e) reg_fence(sr[q][e]);
        const int valid = kb == NB - 1 ? L - kb * BN : BN;
        if (valid < BN) {
#pragma unroll
          for (int q = 0; q < 2; ++q)
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int key = (q * 8 + (e >> 2)) * 8 + 2 * j4 + (e & 1);
              if (key >= valid) sr[q][e] = __float_as_uint(-INFINITY);
            }
        }
        float xa = -INFINITY, xb = -INFINITY, ya = -INFINITY, yb = -INFINITY;
#pragma unroll
        for (int q = 0; q < 2; ++q)
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            xa = max3(xa, __uint_as_float(sr[q][e]), __uint_as_float(sr[q][e + 1]));
            ya = max3(ya, __uint_as_float(sr[q][e + 2]), __uint_as_float(sr[q][e + 3]));
            xb = max3(xb, __uint_as_float(sr[q][e + 4]), __uint_as_float(sr[q][e + 5]));
            yb = max3(yb, __uint_as_float(sr[q][e + 6]), __uint_as_float(sr[q][e + 7]));
          }
        float mxA = fmaxf(xa, xb), mxB = fmaxf(ya, yb);
        mxA = fmaxf(mxA, __shfl_xor_sync(0xffffffffu, mxA, 1));
        mxB = fmaxf(mxB, __shfl_xor_sync(0xffffffffu, mxB, 1));
        mxA = fmaxf(mxA, __shfl_xor_sync(0xffffffffu, mxA, 2));
        mxB = fmaxf(mxB, __shfl_xor_sync(0xffffffffu, mxB, 2));
        const float nA = fmaxf(mA, mxA * sl2), nB = fmaxf(mB, mxB * sl2);
        const bool rsA = nA > mA + kRescaleThreshold, rsB = nB > mB + kRescaleThreshold;
        float fA = 1.f, fB = 1.f;
        if (rsA) {
          fA = ex2_approx(mA - nA);  // 0 when mA is -inf
          lA *= fA;
          kA *= fA;
          mA = nA;
        }
        if (rsB) {
          fB = ex2_approx(mB - nB);
          lB *= fB;
          kB *= fB;
          mB = nB;
        }
        if (nt > 0 && __any_sync(0xffffffffu, rsA || rsB)) {
          // O must hold the previous block's PV before it is rescaled
          if (!(ok = warp_wait(&sh->pv_done[(u - 1) % NS], ((u - 1) / NS) & 1, sh, prm))) break;
          tc_fence_after();
#pragma unroll
          for (int cc = 0; cc < OB_RESCALE * D / 64; ++cc) {  // fused: OK and OR
            uint32_t o[32];
            tmem_ld_16x256b_x8(tO + cc * 64, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              reg_fence(o[e]);
              o[e] = __float_as_uint(__uint_as_float(o[e]) * ((e & 2) ? fB : fA));
            }
            tmem_st_16x256b_x8(tO + cc * 64, o);
          }
          tmem_wait_st();
        }
        const uint64_t negA = f2_pack(mA == -INFINITY ? 0.f : -mA, mA == -INFINITY ? 0.f : -mA);
        const uint64_t negB = f2_pack(mB == -INFINITY ? 0.f : -mB, mB == -INFINITY ? 0.f : -mB);
        uint64_t accA0 = 0ull, accA1 = 0ull, accB0 = 0ull, accB1 = 0ull;
        uint32_t pk[32];  // P columns 4*chunk + j4: {row rA, row rA+8} per chunk
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const uint32_t* c4 = &sr[k >> 3][(k & 7) * 4];
          const uint64_t xA = f2_fma(f2_pack(__uint_as_float(c4[0]), __uint_as_float(c4[1])), scale2, negA);
          const uint64_t xB = f2_fma(f2_pack(__uint_as_float(c4[2]), __uint_as_float(c4[3])), scale2, negB);
          float pa0, pa1, pb0, pb1;
          if ((kPolyPairs >> (2 * k)) & 1u) {
            f2_unpack(exp2_poly(xA), pa0, pa1);
          } else {
            float a0, a1;
            f2_unpack(xA, a0, a1);
            pa0 = ex2_approx(a0);
            pa1 = ex2_approx(a1);
          }
          if ((kPolyPairs >> (2 * k + 1)) & 1u) {
            f2_unpack(exp2_poly(xB), pb0, pb1);
          } else {
            float b0, b1;
            f2_unpack(xB, b0, b1);
            pb0 = ex2_approx(b0);
            pb1 = ex2_approx(b1);
          }
          if (k & 1) {
            accA1 = f2_add(accA1, f2_pack(pa0, pa1));
            accB1 = f2_add(accB1, f2_pack(pb0, pb1));
          } else {
            accA0 = f2_add(accA0, f2_pack(pa0, pa1));
            accB0 = f2_add(accB0, f2_pack(pb0, pb1));
          }
          pk[2 * k] = pack_bf16x2(pa0, pa1);
          pk[2 * k + 1] = pack_bf16x2(pb0, pb1);
        }
        tmem_st_16x128b_x16(tS, pk);
        {
          float a0, a1, b0, b1;
          f2_unpack(f2_add(accA0, accA1), a0, a1);
          f2_unpack(f2_add(accB0, accB1), b0, b1);
          lA += a0 + a1;
          lB += b0 + b1;
          if (kFused && kept) {
            kA += a0 + a1;
            kB += b0 + b1;
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&sh->p_full[b]);
        ++u;
        ++nt;
      }
      if (!ok) break;
      // full row sums, then hand the statistics of this item to the epilogue
      lA += __shfl_xor_sync(0xffffffffu, lA, 1);
      lB += __shfl_xor_sync(0xffffffffu, lB, 1);
      lA += __shfl_xor_sync(0xffffffffu, lA, 2);
      lB += __shfl_xor_sync(0xffffffffu, lB, 2);
      if (kFused) {
        kA += __shfl_xor_sync(0xffffffffu, kA, 1);
        kB += __shfl_xor_sync(0xffffffffu, kB, 1);
        kA += __shfl_xor_sync(0xffffffffu, kA, 2);
        kB += __shfl_xor_sync(0xffffffffu, kB, 2);
      }
      if (i >= 2 && !(ok = warp_wait(&sh->stats_free[sb], ((i - 2) >> 1) & 1, sh, prm))) break;
      float* st = stats + sb * 3 * BM;
      if (j4 == 0) {
        st[rA] = lA;
        st[rA + 8] = lB;
        st[BM + rA] = mA;
        st[BM + rA + 8] = mB;
        if (kFused) {
          st[2 * BM + rA] = kA;
          st[2 * BM + rA + 8] = kB;
        }
      }
      mbar_arrive(&sh->stats_full[sb]);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    setmaxnreg_dec<kRegsEpilogue>();
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    bool ok = true;
    for (int i = 0; ok; ++i) {
      const int w = next_item(i, sh, prm);
      if (w < 0) break;
      const auto it = item_at<kFused, kIntervals>(w, prm);
      const int ob = i % OB;
      const int sb = i & 1;
      if (!(ok = warp_wait(&sh->o_full[ob], (i / OB) & 1, sh, prm))) break;
      if (!(ok = warp_wait(&sh->stats_full[sb], (i >> 1) & 1, sh, prm))) break;
      tc_fence_after();
      const float* st = stats + sb * 3 * BM;
      const float l = st[r];
      const float m_ref = st[BM + r];
      const int grow = it.qb * BM + r;
      // output row: the row map (fused correction path only), checked
      int orow = grow;
      if (!kFused && prm.out_rows && grow < L) {
        orow = __ldg(prm.out_rows + grow);
        if (static_cast<unsigned>(orow) >= static_cast<unsigned>(L)) {
          flag_status(prm, BSA_DEV_BAD_INDEX);
          orow = -1;
        }
      }
      const bool store = grow < L && orow >= 0;
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      const size_t row_elem = (static_cast<size_t>(it.bh) * L + (store ? grow : 0)) * D;
      const size_t out_elem = (static_cast<size_t>(it.bh) * L + (store ? orow : 0)) * D;
      const uint32_t tO = tmem + lane_off + COL_O + ob * D;
      if constexpr (kFused) {
        // dense = (OK + OR) / l, sparse = OK / l_kept.  OK holds data only if
        // some block was kept (l_kept > 0), OR only if some block was not,
        // which is exactly when l differs from l_kept (the two sums add the
        // same terms in the same order otherwise); an accumulator that no PV
        // of this item wrote still holds an earlier item's values.
        const float lk = st[2 * BM + r];
        mbar_arrive(&sh->stats_free[sb]);
        const bool rest = l != lk;
        const bool kept_any = lk > 0.f;
        const float inv_k = lk > 0.f ? 1.f / lk : 0.f;
#pragma unroll
        for (int cc = 0; cc < D / 16; ++cc) {
          uint32_t ok_[16], or_[16];
          tmem_ld16(tO + cc * 16, ok_);
          tmem_ld16(tO + D + cc * 16, or_);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            reg_fence(ok_[e]);
            reg_fence(or_[e]);
          }
          if (cc == D / 16 - 1) {
            // OK and OR have been read out: the next item's PV may overwrite them
            tc_fence_before();
            mbar_arrive(&sh->o_empty[ob]);
          }
          if (store) {
            uint32_t pd[8], ps[8], pr[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              float d0 = kept_any ? __uint_as_float(ok_[2 * e]) : 0.f;
              float d1 = kept_any ? __uint_as_float(ok_[2 * e + 1]) : 0.f;
              const float s0 = d0 * inv_k, s1 = d1 * inv_k;
              if (rest) {
                d0 += __uint_as_float(or_[2 * e]);
                d1 += __uint_as_float(or_[2 * e + 1]);
              }
              pd[e] = pack_bf16x2(d0 * inv_l, d1 * inv_l);
              ps[e] = pack_bf16x2(s0, s1);
              // R = bf16(bf16(O_dense) - bf16(O_sparse))
              pr[e] = pack_bf16x2(__uint_as_float(pd[e] << 16) - __uint_as_float(ps[e] << 16),
                                  __uint_as_float(pd[e] & 0xFFFF0000u) - __uint_as_float(ps[e] & 0xFFFF0000u));
            }
            uint4* od = reinterpret_cast<uint4*>(prm.o + row_elem + cc * 16);
            uint4* os = reinterpret_cast<uint4*>(prm.o2 + row_elem + cc * 16);
            od[0] = make_uint4(pd[0], pd[1], pd[2], pd[3]);
            od[1] = make_uint4(pd[4], pd[5], pd[6], pd[7]);
            os[0] = make_uint4(ps[0], ps[1], ps[2], ps[3]);
            os[1] = make_uint4(ps[4], ps[5], ps[6], ps[7]);
            if (prm.r_out) {
              uint4* orr = reinterpret_cast<uint4*>(prm.r_out + row_elem + cc * 16);
              orr[0] = make_uint4(pr[0], pr[1], pr[2], pr[3]);
              orr[1] = make_uint4(pr[4], pr[5], pr[6], pr[7]);
            }
          }
        }
        if (store) {
          const size_t rr = static_cast<size_t>(it.bh) * L + grow;
          prm.lse[rr] = l > 0.f ? (m_ref + log2f(l)) * 0.69314718055994531f : -INFINITY;
          prm.lse2[rr] = lk > 0.f ? (m_ref + log2f(lk)) * 0.69314718055994531f : -INFINITY;
          if (prm.mass) prm.mass[rr] = l > 0.f ? lk / l : 0.f;  // exactly 1 when every block is kept
        }
      } else {
        const float a = prm.R ? __ldg(prm.alpha + it.bh % prm.H) : 0.f;
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t regs[32];
          tmem_ld32(tO + cc * 32, regs);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) reg_fence(regs[e]);
          if (store) {
            float v[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = l > 0.f ? __uint_as_float(regs[e]) * inv_l : 0.f;
            if (prm.R) {
              // R follows q, k, v; with row gathers, the order of o
              const uint4* rp = reinterpret_cast<const uint4*>(prm.R + (kGather ? out_elem : row_elem) + cc * 32);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const uint4 rv = __ldg(rp + q);
                const uint32_t rw[4] = {rv.x, rv.y, rv.z, rv.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  v[q * 8 + 2 * e] += a * __uint_as_float(rw[e] << 16);
                  v[q * 8 + 2 * e + 1] += a * __uint_as_float(rw[e] & 0xFFFF0000u);
                }
              }
            }
            uint4* op = reinterpret_cast<uint4*>(prm.o + out_elem + cc * 32);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint4 ov;
              ov.x = pack_bf16x2(v[q * 8 + 0], v[q * 8 + 1]);
              ov.y = pack_bf16x2(v[q * 8 + 2], v[q * 8 + 3]);
              ov.z = pack_bf16x2(v[q * 8 + 4], v[q * 8 + 5]);
              ov.w = pack_bf16x2(v[q * 8 + 6], v[q * 8 + 7]);
              op[q] = ov;
            }
          }
        }
        if (store)
          prm.lse[static_cast<size_t>(it.bh) * L + orow] =
              l > 0.f ? (m_ref + log2f(l)) * 0.69314718055994531f : -INFINITY;
        tc_fence_before();
        mbar_arrive(&sh->o_empty[ob]);
        mbar_arrive(&sh->stats_free[sb]);
      }
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0 && sh->joined) {
    // this CTA has made its final fetch (or given up): leave the slot
    sched_leave(&g_sched[prm.sched_slot], launch_tag(), prm);
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

// [BH * L, D] bf16 as a 2-D tensor whose box is one row of 64 columns, for
// 4-row gathers.
bool make_map_rows(CUtensorMap* m, const void* base, int D, long long rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2};
  const cuuint32_t box[2] = {64, 1};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [BH, L, D] E4M3 (raw bytes) as a 3-D tensor; box = 128 columns (128 bytes) x rows x 1.
bool make_map8(CUtensorMap* m, const void* base, int D, int L, int BH, int box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(L), static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(L) * D};
  const cuuint32_t box[3] = {128, static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, bool kFused, bool kF8 = false, bool kGather = false, bool kIntervals = false>
int run(const bsa_shape& s, const AttnArgs& a, cudaStream_t st) {
  using C = Cfg<D, kF8>;
  if (smem_opt_in(reinterpret_cast<const void*>(sparse_attn_tile_kernel<D, kFused, kF8, kGather, kIntervals>),
                  C::SMEM_BYTES) !=
      cudaSuccess)
    return BSA_ECUDA;
  const int BH = s.B * s.H;
  const long long n_rows = static_cast<long long>(BH) * s.L;
  if (kGather && n_rows >= (1ll << 31)) return BSA_ESHAPE;  // row coordinates are int32
  CUtensorMap mq, mk, mv;
  if (kGather) {
    if (!make_map_rows(&mq, a.q, D, n_rows) || !make_map_rows(&mk, a.k, D, n_rows) ||
        !make_map_rows(&mv, a.v, D, n_rows))
      return BSA_ECUDA;
  } else if (kF8) {
    if (!make_map8(&mq, a.q8, D, s.L, BH, BM) || !make_map8(&mk, a.k8, D, s.L, BH, BN)) return BSA_ECUDA;
  } else if (!make_map(&mq, a.q, D, s.L, BH, BM) || !make_map(&mk, a.k, D, s.L, BH, BN)) {
    return BSA_ECUDA;
  }
  if (!kGather && !make_map(&mv, a.v, D, s.L, BH, BN)) return BSA_ECUDA;
  Params prm;
  prm.kept_idx = a.kept_idx;
  prm.kept_cnt = a.kept_cnt;
  prm.R = a.R;
  prm.alpha = a.alpha;
  prm.o = a.o;
  prm.lse = a.lse;
  prm.o2 = a.o2;
  prm.lse2 = a.lse2;
  prm.r_out = a.r_out;
  prm.mass = a.mass;
  prm.out_rows = a.out_rows;
  prm.status = a.status;
  prm.q_scale = a.q_scale;
  prm.k_scale = a.k_scale;
  prm.in_rows = a.in_rows;
  prm.intervals = a.intervals;
  prm.n_int = a.n_int;
  prm.W = a.W;
  prm.n_rows = static_cast<int>(n_rows < (1ll << 31) ? n_rows : 0);
  prm.H = s.H;
  prm.L = s.L;
  prm.NB = n_blocks(s.L, s.blk);
  prm.NT = prm.NB;  // one work item per 128-token query block
  prm.n_work = BH * prm.NT;
  prm.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(D)));
  prm.dense = a.kept_idx == nullptr && a.intervals == nullptr;
  static std::atomic<unsigned int> launches{0};
  prm.sched_slot = static_cast<int>(launches.fetch_add(1u) % kSchedSlots);
  const int sms = sm_count();
  const int grid = prm.n_work < sms ? prm.n_work : sms;
  sparse_attn_tile_kernel<D, kFused, kF8, kGather, kIntervals><<<grid, kThreads, C::SMEM_BYTES, st>>>(mq, mk, mv,
                                                                                                      prm);
  return cudaGetLastError() == cudaSuccess ? BSA_OK : BSA_ECUDA;
}

}  // namespace tile_attn

int launch_sparse_attn_tile(const bsa_shape& s, const AttnArgs& a, cudaStream_t st) {
  if (s.blk != 128) return BSA_ESHAPE;
  if (a.intervals) {
    if (a.o2 || a.q8 || a.in_rows) return BSA_ESHAPE;
    if (s.D == 128) return tile_attn::run<128, false, false, false, true>(s, a, st);
    if (s.D == 64) return tile_attn::run<64, false, false, false, true>(s, a, st);
    return BSA_ESHAPE;
  }
  if (a.in_rows) {
    if (s.D == 128 && !a.o2 && !a.q8) return tile_attn::run<128, false, false, true>(s, a, st);
    return BSA_ESHAPE;
  }
  if (a.q8) {
    if (s.D == 128 && !a.o2) return tile_attn::run<128, false, true>(s, a, st);
    return BSA_ESHAPE;
  }
  if (a.o2) {
    if (s.D == 128) return tile_attn::run<128, true>(s, a, st);
    if (s.D == 64) return tile_attn::run<64, true>(s, a, st);
    return BSA_ESHAPE;
  }
  if (s.D == 128) return tile_attn::run<128, false>(s, a, st);
  if (s.D == 64) return tile_attn::run<64, false>(s, a, st);
  return BSA_ESHAPE;
}

}  // namespace bsa

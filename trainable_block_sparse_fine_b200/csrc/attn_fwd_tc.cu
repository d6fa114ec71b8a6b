// Block-sparse attention forward on tcgen05 (bf16 in, fp32 accumulate), head_dim 128.
// Eq. 12 of "Improving Video Sparse Attention with Fine-grained Router and Sparse Rebasing",
// with the attention definition of its §2.1: per query tile, softmax over the tokens of the
// KV tiles its router selected.
//
// Design for sm_100a. Gathered K/V tiles reach shared memory through TMA and are read once by
// the tensor core, so shared-memory bandwidth (128 B/clk/SM, shared by TMA writes and MMA
// operand reads) is the binding resource. Both GEMMs therefore take their A operand from
// tensor memory and only their B operand from shared memory:
//   S  [64 q, 128 kv] = Q  . [K_j1; K_j2]^T   A = Q (TMEM, written once per tile), B = K (K-major)
//   O  [64 q, 128 d] += P  . [V_j1; V_j2]     A = P (TMEM, written by the softmax), B = V (MN-major)
// M=64 tiles occupy half of the TMEM lanes (lanes 0-15 of each 32-lane quarter), so two query
// tiles ("slots") share the same TMEM columns: slot 0 at lane offset 0, slot 1 at offset 16.
//
// CTA (persistent): warps 0-3 run the softmax of slot 0, warps 4-7 of slot 1. A warp owns 16
// rows of its slot; the 16x64b TMEM access gives each row to a pair of threads (even / odd
// columns), so row max and row sum need one shuffle and no block-level barrier. The two slots
// are independent pipelines sharing only the tensor pipe: warps 8 and 10 load the K and V
// blocks of slot 0 and slot 1 into the slot's own ring, warps 9 and 11 issue its MMAs. The ring
// holds K and V blocks alike, in the slot's op order, so each block is requested three ops ahead
// of its MMA: V(i) as soon as S(i) has read K(i), K(i+1) once O(i-2) has read V(i-2). The running
// max is raised (with an O rescale in TMEM) only when a row's new maximum exceeds it by more
// than 2^8.
//
// kMode selects the key mask: 0 = none (the fine branch, Eq. 12); 1 = keys at or beyond
// `kv_valid` tokens of a head are padding (a sequence whose last tile is partly padding, such as
// the coarse branch's N pooled rows, Eq. 1-3); 2 = a grid the tile does not divide, with the
// real tokens of every tile in `tmask` (§2.2 "Kernel Implementation"): padding keys are masked
// and padding query rows are written as o = 0, lse = -inf. Every listed tile must hold at least
// one valid key.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace vsa2 {
namespace {

constexpr int FT = 384;            // 12 warps
constexpr uint32_t TILE_B = 8192;  // one 64x64 bf16 box (64 rows x 128 B)
constexpr uint32_t BLK_B = 32768;  // K or V block: [half0: tile A, tile B][half1: tile A, tile B]
constexpr int RST = 3;             // ring stages per slot (K and V blocks in op order)
constexpr int kLead = 1;           // S(k) is issued before O(k - 1) and after O(k - 2), which reads
                                   // the P that S(k) overwrites: the lead must stay 1

// Each slot has its own ring (one producer, one consumer, both in the slot's op order), so
// every barrier wait is for the phase in progress or the one just completed.
constexpr uint32_t OFF_RING = 0;                           // [slot][RST] blocks
constexpr int IDXCAP = 256;                                // KV indices of a row kept in shared memory
constexpr uint32_t OFF_IDX = OFF_RING + 2 * RST * BLK_B;   // [slot][2 rows][IDXCAP] int32
constexpr uint32_t OFF_BAR = OFF_IDX + 2 * 2 * IDXCAP * 4;
constexpr uint32_t OFF_FLAG = OFF_BAR + 512;
constexpr int QD = 4;                                       // item queue entries per slot
constexpr uint32_t OFF_IQ = OFF_FLAG + 64;                  // [slot][QD] items, then [slot][2] hand-over
constexpr uint32_t SMEM_USED = OFF_IQ + (2 * QD + 2 * 2) * 4;
constexpr uint32_t SMEM_DYN = SMEM_USED + 1024;
static_assert(SMEM_DYN <= 232448, "shared memory budget");

// TMEM columns (each region used by both slots through the lane halves). The softmax writes
// P(n) as bf16 over the first 64 columns of the S buffer it read S(n) from, so P is double
// buffered with S: the softmax of block n+1 never waits for the P.V MMA of block n. S(n+2)
// overwrites that buffer only after O(n) has read P(n): the MMA issuer issues S(n+2) after O(n),
// and the tensor pipe runs one thread's MMAs in order.
constexpr uint32_t TM_S = 0;      // two S / P buffers of 128 fp32 columns
constexpr uint32_t TM_Q = 256;    // Q: 128 bf16 = 64 columns
constexpr uint32_t TM_O = 320;    // O: 128 fp32 columns
constexpr uint32_t TM_COLS = 512;
constexpr float kThresh = 8.0f;   // log2 headroom before the running max must move

struct Bars {
  uint64_t full[2][RST], empty[2][RST];                                    // [slot][stage]
  uint64_t sfull[2][2], sfree[2][2];                                       // [slot][buffer]
  uint64_t pfull[2][2], pvdone[2][2], qready[2];  // pfull, pvdone: [slot][block parity]
  uint64_t done[2];
  uint64_t iqfull[2][QD], iqempty[2][QD];  // [slot][entry]: the slot's item queue
};
static_assert(sizeof(Bars) <= 512, "barrier area");

struct Row {
  int beg, len;
};
// Sanitised CSR row of query tile i of head bh; every role reads it the same way.
__device__ __forceinline__ Row load_row(const int32_t* kv_off, int bh, int i, int N, int cap, const DevCtx& ctx,
                                        bool report) {
  int b = kv_off[(size_t)bh * (N + 1) + i];
  int e = kv_off[(size_t)bh * (N + 1) + i + 1];
  if (b < 0 || e < b || e > cap || e - b > N) {
    if (report) set_error(ctx.err, VSA2_ERR_BAD_INDEX);
    return Row{0, 0};
  }
  return Row{b, e - b};
}

// Per-slot op stream: items (b*h, query tile) come from a global counter in head-major order, one
// at a time, to whichever slot's producer asks next (the per-sequence TopK gives rows of unequal
// length, so a fixed assignment leaves some slots finishing late). The producer passes each item
// to its slot's MMA issuer and softmax warps through a queue in shared memory. For a tile of n
// blocks the ops are S0, S1, O0, S2, O1, ..., O(n-1); the producer and the MMA issuer walk them in
// the same order.
struct SlotSeq {
  int kq;  // queue entries taken
  int bh, qt, nblk, len, beg;
  int s_next, o_next;
  int tile;  // non-empty tiles started so far
  bool active;
  __device__ void init() {
    kq = 0;
    nblk = 0;
    s_next = o_next = 0;
    tile = 0;
    active = true;
  }
};

// 0 = none, 1 = S op, 2 = O op; *blk = block index within the tile. The next item comes from the
// slot's queue (entry kq % QD); -1 ends the stream.
__device__ __forceinline__ int next_op(SlotSeq& q, int* blk, const int32_t* kv_off, int N, int cap,
                                       const DevCtx& ctx, const volatile int* iq, uint64_t* iqfull,
                                       uint64_t* iqempty, volatile int* abort) {
  while (q.active) {
    if (q.s_next < q.nblk && q.s_next <= q.o_next + kLead) {
      *blk = q.s_next++;
      return 1;
    }
    if (q.o_next < q.nblk) {
      *blk = q.o_next++;
      return 2;
    }
    const int e = q.kq % QD;
    int item = -1;
    if (mbar_wait(&iqfull[e], (q.kq / QD) & 1, abort, ctx)) item = iq[e];
    mbar_arrive(&iqempty[e]);
    ++q.kq;
    if (item < 0) {
      q.active = false;
      return 0;
    }
    q.bh = item / N;
    q.qt = item - q.bh * N;
    const Row r = load_row(kv_off, q.bh, q.qt, N, cap, ctx, false);
    q.len = r.len;
    q.beg = r.beg;
    q.nblk = (r.len + 1) >> 1;
    q.s_next = q.o_next = 0;
    if (q.nblk > 0) q.tile++;
  }
  return 0;
}

// The gated merge of Eq. 13-14 fused into the epilogue (kGate): O = tanh(g) * O_c_hat[tile] + O_f
// with the gate logit g = (X W_g) of the row and the coarse output row of the query tile; the
// fine output O_f can be written too (the backward forms Delta from it).
struct GateArgs {
  const float* logits;           // [b*h, L] fp32
  const __nv_bfloat16* oc;       // [b*h, N, 128], the coarse branch's output
  __nv_bfloat16* of;             // [b*h, L, 128] or nullptr
};

template <int kMode, bool kGate>
__global__ void __launch_bounds__(FT, 1)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                       const __nv_bfloat16* __restrict__ qg, const int32_t* __restrict__ kv_off,
                       const int32_t* __restrict__ kv_idx, __nv_bfloat16* __restrict__ out, float* __restrict__ lse,
                       int N, int L, int topk, int items, float c2, int kv_valid,
                       const uint64_t* __restrict__ tmask, GateArgs gate, int* __restrict__ work_ctr, DevCtx ctx) {
  extern __shared__ __align__(1024) uint8_t dsm_raw[];
  uint8_t* dsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
  Bars& B = *reinterpret_cast<Bars*>(dsm + OFF_BAR);
  int* flag_sh = reinterpret_cast<int*>(dsm + OFF_FLAG);  // [0] abort, [4] tmem base
  volatile int* abort = flag_sh;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cap = N * topk;

  if (threadIdx.x == 0) {
    flag_sh[0] = 0;
    for (int s = 0; s < 2; ++s) {
      for (int i = 0; i < RST; ++i) mbar_init(&B.full[s][i], 1), mbar_init(&B.empty[s][i], 1);
      for (int b = 0; b < 2; ++b) mbar_init(&B.sfull[s][b], 1), mbar_init(&B.sfree[s][b], 4);
      mbar_init(&B.pfull[s][0], 4);
      mbar_init(&B.pfull[s][1], 4);
      mbar_init(&B.pvdone[s][0], 1);
      mbar_init(&B.pvdone[s][1], 1);
      mbar_init(&B.qready[s], 4);
    }
    mbar_init(&B.done[0], 1);
    mbar_init(&B.done[1], 1);
    for (int s = 0; s < 2; ++s)
      for (int i = 0; i < QD; ++i) mbar_init(&B.iqfull[s][i], 1), mbar_init(&B.iqempty[s][i], 2);
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(reinterpret_cast<uint32_t*>(flag_sh + 4), TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(flag_sh + 4);

  if (warp == 8 || warp == 10) {
    // ------------------------------------------------------------------ TMA producer of slot (warp - 8) / 2
    // K blocks for the slot's S ops and V blocks for its O ops, in the slot's op order. The whole
    // warp copies each item's KV indices into shared memory (cp.async) one item ahead, and its
    // row offsets two items ahead, so that lane 0, which issues the copies, never waits for a
    // global load on its way from one op to the next.
    const int s = (warp - 8) >> 1;
    int32_t* ibuf = reinterpret_cast<int32_t*>(dsm + OFF_IDX) + s * 2 * IDXCAP;
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
    }
    auto row_of = [&](int it) { return it >= 0 ? load_row(kv_off, it / N, it % N, N, cap, ctx, false) : Row{0, 0}; };
    auto copy_row = [&](int it, const Row& r, int b) {  // whole warp
      const int32_t* src = kv_idx + (size_t)(it / N) * cap + r.beg;
      const int n = min(r.len, IDXCAP);
      for (int e = lane; e < n; e += 32)
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(ibuf + b * IDXCAP + e)), "l"(src + e)
                     : "memory");
      asm volatile("cp.async.commit_group;" ::: "memory");
    };
    // Items come from a global counter (dynamic balance across slots). Lane 0 takes one when the
    // warp needs it, two items ahead of the loads, and passes it to the slot's MMA issuer and
    // softmax warps through the queue, in load order; -1 marks the end.
    volatile int* iq = reinterpret_cast<volatile int*>(dsm + OFF_IQ) + s * QD;
    int kq = 0;  // queue entries written
    bool ended = false;
    bool ok = true;
    auto next_id = [&]() -> int {  // whole warp
      if (ended) return -1;
      int id = -1, good = 1;
      if (lane == 0) {
        id = atomicAdd(work_ctr, 1);
        if (id >= items) id = -1;
        const int e = kq % QD;
        if (mbar_wait(&B.iqempty[s][e], ((kq / QD) & 1) ^ 1, abort, ctx)) {
          iq[e] = id;
          mbar_arrive(&B.iqfull[s][e]);
        } else {
          good = 0;
        }
      }
      id = __shfl_sync(0xffffffffu, id, 0);
      good = __shfl_sync(0xffffffffu, good, 0);
      ++kq;
      if (!good) ok = false;
      if (id < 0 || !good) {
        ended = true;
        id = -1;
      }
      return id;
    };
    int item = next_id();
    Row cur = row_of(item);
    if (item >= 0) copy_row(item, cur, 0);
    int nxt_id = next_id();
    Row nxt = row_of(nxt_id);
    int c = 0;  // ring position: blocks requested so far
    for (int b = 0; ok && item >= 0; b ^= 1) {
      asm volatile("cp.async.wait_all;" ::: "memory");  // this item's indices (copied an item ago)
      __syncwarp();
      if (nxt_id >= 0 && nxt.len > 0) copy_row(nxt_id, nxt, b ^ 1);
      const int nn_id = next_id();
      const Row nn = row_of(nn_id);  // used when the next item starts
      if (lane == 0) {
        const int bh = item / N;
        const int32_t* gidx = kv_idx + (size_t)bh * cap + cur.beg;
        const int32_t* sidx = ibuf + b * IDXCAP;
        const int nblk = (cur.len + 1) >> 1;
        int s_next = 0, o_next = 0;
        while (o_next < nblk) {
          int blk;
          bool k_op;
          if (s_next < nblk && s_next <= o_next + kLead) {
            blk = s_next++;
            k_op = true;
          } else {
            blk = o_next++;
            k_op = false;
          }
          const int ntile = min(2, cur.len - 2 * blk);
          int j[2] = {0, 0};
#pragma unroll
          for (int tt = 0; tt < 2; ++tt) {
            if (tt >= ntile) break;
            const int e = 2 * blk + tt;
            int v = e < IDXCAP ? sidx[e] : gidx[e];
            if (v < 0 || v >= N) {
              if (ctx.flags & VSA2_FLAG_VALIDATE) set_error(ctx.err, VSA2_ERR_BAD_INDEX);
              v = min(max(v, 0), N - 1);
            }
            j[tt] = v;
          }
          const int st = c % RST;
          uint64_t* full = &B.full[s][st];
          uint8_t* dst = dsm + OFF_RING + (s * RST + st) * BLK_B;
          if (!(ok = mbar_wait(&B.empty[s][st], ((c / RST) & 1) ^ 1, abort, ctx))) break;
          mbar_arrive_expect_tx(full, ntile * 2 * TILE_B);
          for (int tt = 0; tt < ntile; ++tt)
            for (int h = 0; h < 2; ++h)
              tma_load_2d(dst + h * 2 * TILE_B + tt * TILE_B, k_op ? &tm_k : &tm_v, h * 64, bh * L + j[tt] * 64,
                          full);
          ++c;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0 && ok;
      item = nxt_id;
      cur = nxt;
      nxt_id = nn_id;
      nxt = nn;
    }
    asm volatile("cp.async.wait_all;" ::: "memory");  // no copy outlives the CTA
    if (lane == 0 && *abort) {  // let copies still in flight land before the CTA exits
      for (int cc = max(0, c - RST); cc < c; ++cc)
        mbar_wait_drain(&B.full[s][cc % RST], (cc / RST) & 1, ctx.timeout_ns);
    }
  } else if (warp == 9 || warp == 11) {
    // ------------------------------------------------------------------ MMA issuer of slot (warp - 9) / 2
    if (lane == 0) {
      const int s = (warp - 9) >> 1;
      constexpr uint32_t id_s = idesc_bf16_f32(64, 128, false, false);
      constexpr uint32_t id_o = idesc_bf16_f32(64, 128, false, true);
      const uint32_t lanes = (uint32_t)(16 * s) << 16;
      SlotSeq sq;
      sq.init();
      const volatile int* iq = reinterpret_cast<const volatile int*>(dsm + OFF_IQ) + s * QD;
      int kc = 0, vc = 0;  // S and O blocks issued
      int c = 0;           // ring position
      bool ok = true;
      while (ok && sq.active) {
        int blk;
        const int op = next_op(sq, &blk, kv_off, N, cap, ctx, iq, B.iqfull[s], B.iqempty[s], abort);
        if (op == 1) {
          if (blk == 0 && !(ok = mbar_wait(&B.qready[s], (sq.tile - 1) & 1, abort, ctx))) break;
          const int st = c % RST;
          if (!(ok = mbar_wait(&B.full[s][st], (c / RST) & 1, abort, ctx))) break;
          if (!(ok = mbar_wait(&B.sfree[s][kc & 1], ((kc >> 1) & 1) ^ 1, abort, ctx))) break;
          tc_fence_after();
          const uint32_t ka = smem_u32(dsm + OFF_RING + (s * RST + st) * BLK_B);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16_ts(tmem + lanes + TM_S + (kc & 1) * 128, tmem + lanes + TM_Q + 8 * kk,
                        sdesc_sw128(ka + (kk >> 2) * 2 * TILE_B + (kk & 3) * 32, 16, 1024), id_s, kk > 0);
          mma_commit(&B.empty[s][st]);
          mma_commit(&B.sfull[s][kc & 1]);
          ++kc;
          ++c;
        } else if (op == 2) {
          const int st = c % RST;
          if (!(ok = mbar_wait(&B.full[s][st], (c / RST) & 1, abort, ctx))) break;
          if (!(ok = mbar_wait(&B.pfull[s][vc & 1], (vc >> 1) & 1, abort, ctx))) break;
          tc_fence_after();
          const uint32_t va = smem_u32(dsm + OFF_RING + (s * RST + st) * BLK_B);
          const int ksteps = (2 * blk + 1 == sq.len) ? 4 : 8;
          for (int kk = 0; kk < ksteps; ++kk)
            mma_bf16_ts(tmem + lanes + TM_O, tmem + lanes + TM_S + (vc & 1) * 128 + 8 * kk,
                        sdesc_sw128(va + kk * 2048, 2 * TILE_B, 1024), id_o, (blk > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&B.empty[s][st]);
          mma_commit(&B.pvdone[s][vc & 1]);
          ++vc;
          ++c;
        }
      }
      mma_commit(&B.done[s]);
      mbar_wait_drain(&B.done[s], 0, ctx.timeout_ns);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------------ softmax, one slot per warpgroup
    const int s = warp >> 2;
    const int w = warp & 3;                        // TMEM lane quarter
    const int bar_id = 1 + s;
    const int r16 = 8 * (lane & 1) + (lane >> 2);  // row within this warp's 16
    const int par_c = (lane >> 1) & 1;             // even / odd columns
    const int row = 16 * w + r16;                  // row within the query tile
    const uint32_t tl = tmem + ((uint32_t)(32 * w + 16 * s) << 16);
    int g = 0;  // blocks processed by this slot
    const volatile int* iq = reinterpret_cast<const volatile int*>(dsm + OFF_IQ) + s * QD;
    volatile int* cur_item = reinterpret_cast<volatile int*>(dsm + OFF_IQ) + 2 * QD + 2 * s;  // [kq parity]
    for (int kq = 0;; ++kq) {
      // the slot's first warp takes the next queue entry and hands it to the slot's 4 warps; the
      // hand-over slot alternates with the entry's parity, so it is rewritten only after every
      // warp passed the next barrier
      if (w == 0 && lane == 0) {
        const int e = kq % QD;
        int id = -1;
        if (mbar_wait(&B.iqfull[s][e], (kq / QD) & 1, abort, ctx)) id = iq[e];
        mbar_arrive(&B.iqempty[s][e]);
        cur_item[kq & 1] = id;
      }
      named_bar_sync(bar_id, 128);
      const int item = cur_item[kq & 1];
      if (item < 0) break;
      const int bh = item / N, qt = item - bh * N;
      const Row rw = load_row(kv_off, bh, qt, N, cap, ctx, w == 0 && lane == 0);
      const int nblk = (rw.len + 1) >> 1;
      const size_t tok = (size_t)bh * L + (size_t)qt * 64 + row;
      if (nblk == 0) {
        // empty selection: o = 0, lse = -inf (each thread of a pair writes half the row); with the
        // gate the output is the coarse term alone
        uint4* o4 = reinterpret_cast<uint4*>(out + tok * 128 + par_c * 64);
        if constexpr (kGate) {
          const float gt = tanhf(__ldg(gate.logits + tok));
          const uint4* c4 = reinterpret_cast<const uint4*>(gate.oc + ((size_t)bh * N + qt) * 128 + par_c * 64);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const uint4 c = __ldg(c4 + e);
            const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
            uint32_t r[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
              r[u] = pack_bf16(gt * __uint_as_float(cw[u] << 16), gt * __uint_as_float(cw[u] & 0xffff0000u));
            o4[e] = make_uint4(r[0], r[1], r[2], r[3]);
          }
          if (gate.of) {
            uint4* f4 = reinterpret_cast<uint4*>(gate.of + tok * 128 + par_c * 64);
#pragma unroll
            for (int e = 0; e < 8; ++e) f4[e] = make_uint4(0, 0, 0, 0);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) o4[e] = make_uint4(0, 0, 0, 0);
        }
        if (par_c == 0) lse[tok] = -INFINITY;
        continue;
      }
      {
        // Q row into TMEM (A operand of S): packed words j = 2i + par_c hold d = 2j, 2j+1
        uint32_t qv[32];
        const uint2* src = reinterpret_cast<const uint2*>(qg + tok * 128);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const uint2 v = __ldg(src + i);
          qv[i] = par_c ? v.y : v.x;
        }
        tmem_st16x64b_x32(tl + TM_Q, qv);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&B.qready[s]);
      }
      float m = -INFINITY, l = 0.f;
      for (int n = 0; n < nblk; ++n, ++g) {
        const bool half = (2 * n + 1 == rw.len);
        mbar_wait(&B.sfull[s][g & 1], (g >> 1) & 1, abort, ctx);
        tc_fence_after();
        uint32_t x[64];
        tmem_ld16x64b_x64(tl + TM_S + (g & 1) * 128, x);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&B.sfree[s][g & 1]);
        if constexpr (kMode == 1) {
          // keys of the block's two tiles at or beyond kv_valid get a score of -inf
          const int32_t* ix = kv_idx + (size_t)bh * cap + rw.beg + 2 * n;
          const int v1 = kv_valid - 64 * __ldg(ix);
          const int v2 = half ? 64 : kv_valid - 64 * __ldg(ix + 1);
          if (v1 < 64 || v2 < 64) {
#pragma unroll
            for (int i = 0; i < 64; ++i)
              if (((2 * i + par_c) & 63) >= (i < 32 ? v1 : v2)) x[i] = __float_as_uint(-INFINITY);
          }
        } else if constexpr (kMode == 2) {
          // padding tokens of the block's two tiles get a score of -inf
          const int32_t* ix = kv_idx + (size_t)bh * cap + rw.beg + 2 * n;
          const uint64_t m1 = __ldg(tmask + min(max(__ldg(ix), 0), N - 1));
          const uint64_t m2 = half ? ~0ull : __ldg(tmask + min(max(__ldg(ix + 1), 0), N - 1));
          if ((m1 & m2) != ~0ull) {
#pragma unroll
            for (int i = 0; i < 64; ++i)
              if (!(((i < 32 ? m1 : m2) >> ((2 * i + par_c) & 63)) & 1ull)) x[i] = __float_as_uint(-INFINITY);
          }
        }
        // columns 2i + par_c; in a half block only the first 64 columns are real
        float mx = __uint_as_float(x[0]);
        if (!half) {
#pragma unroll
          for (int i = 1; i < 63; i += 2) mx = fmax3(mx, __uint_as_float(x[i]), __uint_as_float(x[i + 1]));
          mx = fmaxf(mx, __uint_as_float(x[63]));
        } else {
#pragma unroll
          for (int i = 1; i < 31; i += 2) mx = fmax3(mx, __uint_as_float(x[i]), __uint_as_float(x[i + 1]));
          mx = fmaxf(mx, __uint_as_float(x[31]));
        }
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2)) * c2;
        float alpha = 1.f;
        const bool raise = mx > m + kThresh;
        if (raise) {
          alpha = (m == -INFINITY) ? 0.f : ex2(m - mx);
          m = mx;
          l *= alpha;
        }
        if (__any_sync(0xffffffffu, raise && n > 0)) {
          // O holds blocks 0..n-1 of this tile: scale the raised rows once the last O MMA is done
          mbar_wait(&B.pvdone[s][(g - 1) & 1], ((g - 1) >> 1) & 1, abort, ctx);
          tc_fence_after();
          uint32_t o[64];
          tmem_ld16x64b_x64(tl + TM_O, o);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 64; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st16x64b_x64(tl + TM_O, o);
          tmem_st_wait();
        }
        // probabilities (<= 2^8), partial row sum, pack bf16 pairs of adjacent columns:
        // the pair partner holds the neighbouring column, so swap half of the values
        // the two columns of a step go through packed fp32 math (one FFMA2, one FADD2)
        uint32_t pk[32];
        const uint32_t perm = pair_perm(par_c);
        const float2 cc = make_float2(c2, c2), nm = make_float2(-m, -m);
        float2 ls = make_float2(0.f, 0.f);
#pragma unroll
        for (int i2 = 0; i2 < 32; ++i2) {
          const float2 arg =
              __ffma2_rn(make_float2(__uint_as_float(x[2 * i2]), __uint_as_float(x[2 * i2 + 1])), cc, nm);
          float pa = ex2(arg.x), pb = ex2(arg.y);
          if (half && i2 >= 16) pa = pb = 0.f;
          ls = __fadd2_rn(ls, make_float2(pa, pb));
          // even thread: word 2*i2 = (col 4*i2, 4*i2+1); odd thread: word 2*i2+1 = (4*i2+2, 4*i2+3)
          pk[i2] = pair_pack_bf16(pa, pb, perm);
        }
        l += ls.x + ls.y;
        // P over the S buffer just read (its S values are in registers)
        tmem_st16x64b_x32(tl + TM_S + (g & 1) * 128, pk);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&B.pfull[s][g & 1]);
      }
      // ---- epilogue: last O block done -> normalise and store
      mbar_wait(&B.pvdone[s][(g - 1) & 1], ((g - 1) >> 1) & 1, abort, ctx);
      tc_fence_after();
      l += __shfl_xor_sync(0xffffffffu, l, 2);
      float inv = 1.f / l;
      float lse_row = (m + __log2f(l)) * 0.6931471805599453f;
      uint32_t o[64];
      tmem_ld16x64b_x64(tl + TM_O, o);
      tmem_ld_wait();
      if constexpr (kMode == 2) {
        if (!((__ldg(tmask + qt) >> row) & 1ull)) {  // a padding query row: o = 0, lse = -inf
#pragma unroll
          for (int i = 0; i < 64; ++i) o[i] = 0u;
          inv = 0.f;
          lse_row = -INFINITY;
        }
      }
      if (par_c == 0) lse[tok] = lse_row;
      // o[i] = O[row][2i + par_c]; swap so each thread holds adjacent pairs, then 4-byte stores
      uint32_t* dst = reinterpret_cast<uint32_t*>(out + tok * 128);
      if constexpr (kGate) {
        // word w = 2*i2 + par_c holds columns 2w, 2w+1: O_f there in fp32, then the gated sum
        const float gt = tanhf(__ldg(gate.logits + tok));
        const uint32_t* ocw = reinterpret_cast<const uint32_t*>(gate.oc + ((size_t)bh * N + qt) * 128);
        uint32_t* fdst = gate.of ? reinterpret_cast<uint32_t*>(gate.of + tok * 128) : nullptr;
#pragma unroll
        for (int i2 = 0; i2 < 32; ++i2) {
          const float a = __uint_as_float(o[2 * i2]) * inv, b = __uint_as_float(o[2 * i2 + 1]) * inv;
          const float send = par_c ? a : b;
          const float recv = __shfl_xor_sync(0xffffffffu, send, 2);
          const float lo = par_c ? recv : a, hi = par_c ? b : recv;
          const int wd = 2 * i2 + par_c;
          const uint32_t c = __ldg(ocw + wd);
          dst[wd] = pack_bf16(fmaf(gt, __uint_as_float(c << 16), lo), fmaf(gt, __uint_as_float(c & 0xffff0000u), hi));
          if (fdst) fdst[wd] = pack_bf16(lo, hi);
        }
      } else {
#pragma unroll
        for (int i2 = 0; i2 < 32; ++i2) {
          const float a = __uint_as_float(o[2 * i2]) * inv, b = __uint_as_float(o[2 * i2 + 1]) * inv;
          const float send = par_c ? a : b;
          const float recv = __shfl_xor_sync(0xffffffffu, send, 2);
          dst[2 * i2 + par_c] = par_c ? pack_bf16(recv, b) : pack_bf16(a, recv);
        }
      }
      // leave together if any wait of this CTA has expired
      if (named_bar_or(bar_id, 128, *abort != 0)) break;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, TM_COLS);
  }
}

}  // namespace

bool make_tmap_2d_bf16(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint32_t box_cols,
                       uint32_t box_rows);

namespace {
template <int kMode, bool kGate = false>
vsa2_status launch_fwd_tc(const Dims& d, const void* q, const void* k, const void* v, int topk,
                          const int32_t* kv_off, const int32_t* kv_idx, void* o, float* lse, char* ws, int kv_valid,
                          const uint64_t* tmask, cudaStream_t s, GateArgs gate = GateArgs{nullptr, nullptr, nullptr}) {
  CUtensorMap tk, tv;
  const uint64_t rows = (uint64_t)d.BH * d.L;
  if (!make_tmap_2d_bf16(&tk, k, 128, rows, 64, 64) || !make_tmap_2d_bf16(&tv, v, 128, rows, 64, 64))
    return tmap_fail("tensor map encoding for the attention operands failed");
  DevCtx ctx{reinterpret_cast<int*>(ws), d.timeout_ns, d.flags};
  const int items = d.BH * d.N;
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = std::max(1, std::min(sms, (items + 1) / 2));
  const float c2 = 1.4426950408889634f / sqrtf(128.f);
  auto kern = attn_fwd_tc_kernel<kMode, kGate>;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_DYN);
  // the item counter the CTAs' producers draw from, in the workspace header
  int* ctr = reinterpret_cast<int*>(ws + kWsWorkCounter);
  if (cudaMemsetAsync(ctr, 0, sizeof(int), s) != cudaSuccess) return cuda_fail("attn_fwd_tc: item counter reset");
  kern<<<grid, FT, SMEM_DYN, s>>>(tk, tv, (const __nv_bfloat16*)q, kv_off, kv_idx, (__nv_bfloat16*)o, lse, d.N,
                                  (int)d.L, topk, items, c2, kv_valid, tmask, gate, ctr, ctx);
  return check_launch("attn_fwd_tc");
}
}  // namespace

vsa2_status attn_fwd_tc(const Dims& d, const void* q, const void* k, const void* v, int topk, const int32_t* kv_off,
                        const int32_t* kv_idx, void* o, float* lse, char* ws, cudaStream_t s) {
  if (d.padded) {
    uint64_t* tmask = reinterpret_cast<uint64_t*>(ws + ws_layout(d).tmask);
    if (launch_tile_masks(d, tmask, s) != VSA2_OK) return VSA2_ERR_CUDA;
    return launch_fwd_tc<2>(d, q, k, v, topk, kv_off, kv_idx, o, lse, ws, (int)d.L, tmask, s);
  }
  return launch_fwd_tc<0>(d, q, k, v, topk, kv_off, kv_idx, o, lse, ws, (int)d.L, nullptr, s);
}

vsa2_status attn_fwd_tc_gated(const Dims& d, const void* q, const void* k, const void* v, int topk,
                              const int32_t* kv_off, const int32_t* kv_idx, const float* gate_logits, const void* oc,
                              void* o, float* lse, void* o_f, char* ws, cudaStream_t s) {
  const GateArgs g{gate_logits, (const __nv_bfloat16*)oc, (__nv_bfloat16*)o_f};
  if (d.padded) {
    uint64_t* tmask = reinterpret_cast<uint64_t*>(ws + ws_layout(d).tmask);
    if (launch_tile_masks(d, tmask, s) != VSA2_OK) return VSA2_ERR_CUDA;
    return launch_fwd_tc<2, true>(d, q, k, v, topk, kv_off, kv_idx, o, lse, ws, (int)d.L, tmask, s, g);
  }
  return launch_fwd_tc<0, true>(d, q, k, v, topk, kv_off, kv_idx, o, lse, ws, (int)d.L, nullptr, s, g);
}

vsa2_status attn_fwd_tc_masked(const Dims& d, const void* q, const void* k, const void* v, int topk,
                               const int32_t* kv_off, const int32_t* kv_idx, void* o, float* lse, char* ws,
                               int kv_valid, cudaStream_t s) {
  return launch_fwd_tc<1>(d, q, k, v, topk, kv_off, kv_idx, o, lse, ws, kv_valid, nullptr, s);
}

}  // namespace vsa2

// Prefill lightning indexer for sm_100a: scores every causal (query, key) pair on the tensor
// cores and streams, per query, the keys that can still enter its top-k into that query's
// candidate buffer in the workspace; prefill_finish_kernel (topk.cu) then takes the exact top-k
// of each buffer. The L x L score matrix is never stored.
//
// One persistent CTA per SM walks query blocks (heaviest first, snake order over CTAs). For a
// block of QB queries it streams the causal key range in tiles of 128 keys:
//   warp 0      TMA producer: the block's Q rows (two 256-row B operands) once, then one
//               [128 keys x d] FP8 K tile per pipeline stage;
//   warp 1      one thread issues tcgen05.mma kind::f8f6f4 (M = 128 keys, N = queries x H
//               heads, K = d) into FP32 accumulators in TMEM. The 512 TMEM columns hold four
//               128-column accumulators in the sample and lean modes and two 256-column ones in
//               the exact mode, so the epilogue of one overlaps the MMAs of the others;
//   warps 4..   four epilogue warps per accumulator (16 in the sample and lean modes, 8 in the
//               exact mode), one per TMEM lane quarter. In the exact mode a thread owns one
//               key (its TMEM lane) and reads all H head dot products of each query; in the
//               sample and lean modes (H = 64) a thread reads 16 lanes x 256 bits at a time,
//               i.e. a quarter of the heads of four keys, and a four-thread reduce-scatter
//               leaves it the full head sum of one key. The epilogue applies ReLU, the head
//               weights, then the query and key scales, masks s > t, and appends the keys it
//               keeps to its warp's segment of the query's buffer (no atomics: the segment's
//               count lives in a register of the warp).
//
// The same kernel runs in three modes:
//   sample  every S-th key only (a strided tensor map), every valid key appended: a uniform
//           sample of each row, from which prefill_sample_threshold_kernel picks a threshold T
//           that at least k keys of the row exceed with overwhelming probability;
//   lean    every key, appended iff key >= T: a compare and an append, nothing else. A query
//           that ends with fewer than min(k, keys in its row) appended keys (T was too high)
//           or a full segment marks its block for the exact mode;
//   exact   no threshold to start with: a nearly full buffer is cut back, by the four warps
//           together, to the keys at or above the bin holding its k-th key (k to k + 128 keys),
//           which also raises the query's threshold. Any key below the threshold has k kept
//           keys above it, so dropping it is exact. Runs on the blocks the lean mode marked,
//           or on every block when k is too small for a useful sample.
//
// ReLU on the FMA pipe: D = q8.k8 with |D| <= d * 448^2 < 2^25, so
// max(D, 0) = 2^25 * sat(D * 2^-25) exactly (power-of-two scalings, no clipping at 1), and
// the 2^25 is folded into the stored head weights.
#include <cstddef>
#include <type_traits>

#include "common.cuh"
#include "internal.h"
#include "select.cuh"

namespace dsa {

template <int H, int D>
struct PCfg {
  static constexpr int QPM = 256 / H;       // queries per MMA (N = 256 columns)
  static constexpr int QB = 2 * QPM;        // queries per block (two accumulators)
  static constexpr int BN = 128;            // keys per tile (MMA M)
  static constexpr int STAGES = (D == 128) ? 4 : 6;
  static constexpr int QTILE = 256 * D;     // bytes of one B operand
  static constexpr int KTILE = BN * D;      // bytes of one A operand
  static constexpr int KSTEPS = D / 32;     // K = 32 per FP8 MMA instruction
  static_assert(D == 64 || D == 128, "d");
  static_assert(H == 8 || H == 64, "H");
};

enum : int { kModeSample = 0, kModeLean = 1, kModeExact = 2 };

// Accumulators and warp roles per mode. The 512 TMEM columns hold NACC accumulators of
// N = 512 / NACC columns ((N / H) queries x H heads); each accumulator is read by four epilogue
// warps, one per TMEM lane quarter. The exact mode has two accumulators (N = 256) and 8
// epilogue warps, so that its two warpgroups' cut-back state fits in shared memory; the sample
// and lean modes have four (N = 128) and 16 epilogue warps: twice the warps to hide the
// TMEM-load and arithmetic latency of the per-key work, and an accumulator's next MMA waits
// only for its own four warps.
template <int H, int MODE>
struct PRoles {
  static constexpr int NACC = MODE == kModeExact ? 2 : 4;
  static constexpr int N = 512 / NACC;                    // MMA N (columns per accumulator)
  static constexpr int EW = 4 * NACC;                     // epilogue warps
  static constexpr int THREADS = 128 + 32 * EW;
  static constexpr int QPW = N / H;                       // queries per accumulator and warp
  static constexpr uint32_t IDESC = make_idesc_f8(128, N);
};

// Selection state of one epilogue warpgroup's cut-backs (exact mode).
struct __align__(16) CutState {
  uint32_t hist[kHistBins];             // zero between cut-backs
  GroupScratch<128> sc;
  uint64_t stage[kPrefillExactCapMax];  // the buffer being cut, contiguous
};

template <int H, int D>
struct PSmem {
  using C = PCfg<H, D>;
  uint8_t q[2][C::QTILE];
  uint8_t k[C::STAGES][C::KTILE];
  float wq[C::QB][H];
  float sq[C::QB];
  uint64_t thr[C::QB];      // per query: lean T; exact running threshold
  uint32_t wcnt[C::QB][4];  // per query: keys in each warp's segment (block end, cut-backs)
  uint32_t cflag[4];        // per query group: queries whose buffer needs a cut-back (exact)
  CutState cut[2];          // per query group of the exact mode (two groups)
  uint64_t kfull[C::STAGES];
  uint64_t kempty[C::STAGES];
  uint64_t qfull, qempty, accfull[4], accempty[4], drain;
  uint32_t tmem_base;
  int abort;
};

using PSmemH64 = PSmem<64, 128>;
using PSmemH8 = PSmem<8, 64>;
static_assert(sizeof(PSmemH64) + 1024 <= 232448, "shared memory of the H=64 kernel");
static_assert(sizeof(PSmemH8) + 1024 <= 232448, "shared memory of the H=8 kernel");
static_assert(offsetof(PSmemH64, wq) % 16 == 0 && offsetof(PSmemH8, wq) % 16 == 0,
              "vectorised weight access");

struct PrefillParams {
  const float* q_scale;
  const float* w;
  const float* k_scale;
  int32_t Lk, q_pos0, Lq, topk;
  int32_t nqb;
  int32_t stride;          // key stride S (sample mode: map row v is key S * v), else 1
  int32_t nkeys;           // rows of the key tensor map (sample mode: ceil(Lk / S))
  uint32_t seg_stride;     // entries between a row's segments (row pitch / 4)
  uint32_t segcap;         // entries a segment may hold in this mode
  uint64_t* cand;          // [Lq][4 * seg_stride]
  uint32_t* counts;        // [Lq][4] keys in each segment after the scan
  uint64_t* thr;           // [Lq] lean: input T; exact: output threshold
  uint32_t* fail_flag;     // [nqb] lean: block needs the exact mode
  int32_t* fail_list;      // [nqb] lean: output list; exact: input list (nullptr: every block)
  uint32_t* fail_count;
  WsHeader* hdr;
  uint64_t budget_ns;
};

// Cut-back of one query's candidate buffer by its warpgroup (128 threads on named barrier
// bar_id). The four segment counts are in wcnt[0..3], segment w at buf + w * seg_stride.
// Stages the segments contiguously in shared memory; with more than k + 128 keys it finds the
// lower edge T of the histogram bin holding the k-th key (k <= count(keys >= T) <= k + 128)
// and keeps the keys >= T, otherwise it keeps every key. The kept keys are written back dealt
// round-robin over the four segments; wcnt and (after a select) *thr are updated. One
// out-of-line copy serves every call site.
__device__ __noinline__ void cut_back(uint64_t* buf, uint32_t seg_stride, uint32_t* wcnt,
                                      uint64_t* thr, CutState* cs, uint32_t k, uint32_t rank,
                                      uint32_t bar_id) {
  const GroupSync<128> gs{bar_id};
  const uint32_t lane = rank & 31u, w = rank >> 5;
  uint32_t n = 0, off = 0;
  for (uint32_t i = 0; i < 4; ++i) {
    const uint32_t c = wcnt[i];
    off += (i < w) ? c : 0u;
    n += c;
  }
  const uint32_t c = wcnt[w];
  const uint64_t* src = buf + w * seg_stride;
  uint64_t* st = cs->stage;
  uint32_t e = lane;
  for (; e + 96 < c; e += 128) {
    const uint64_t a0 = __ldcg(src + e), a1 = __ldcg(src + e + 32), a2 = __ldcg(src + e + 64),
                   a3 = __ldcg(src + e + 96);
    st[off + e] = a0;
    st[off + e + 32] = a1;
    st[off + e + 64] = a2;
    st[off + e + 96] = a3;
  }
  for (; e < c; e += 32) st[off + e] = __ldcg(src + e);
  gs.sync();
  auto key_at = [st](uint32_t i) { return st[i]; };
  uint64_t T = 0;
  if (n > k + 128u) {
    uint32_t cnt;
    T = group_select_threshold<128>(key_at, n, k, k + 128u, rank, cs->hist, cs->sc, gs, &cnt);
  }
  const uint32_t kept = group_compact_ge<128>(
      key_at, n, T,
      [buf, seg_stride](uint32_t pos, uint64_t key) { buf[(pos & 3u) * seg_stride + (pos >> 2)] = key; },
      rank, cs->sc, gs);
  if (rank < 4) wcnt[rank] = (kept + 3u - rank) >> 2;
  if (rank == 0 && T != 0) *thr = T;
  gs.sync();
}

// The head-weighted ReLU sums of one epilogue thread's key for the QPW queries of its
// accumulator: reads QPW * H TMEM columns in 32-column chunks (double-buffered tcgen05.ld)
// and returns, per query, sum_j w'[j] * sat(D_j * 2^-25) with w' = 2^25 w (stored so in wq).
template <int H, int QPW>
__device__ __forceinline__ void head_sums(uint32_t taddr0, const float (*wq)[H], float (&out)[QPW]) {
  constexpr int NCH = QPW * H / 32;
  uint32_t ra[32], rb[32];
  tmem_ld_32x32b_x32(taddr0, ra);
  tmem_wait_ld_regs(ra);
  if constexpr (H == 64) {
    // 64 heads per query: packed FMA over head pairs, four float2 partial sums per query.
    float2 acc[QPW][4];
#pragma unroll
    for (int qi = 0; qi < QPW; ++qi)
#pragma unroll
      for (int a = 0; a < 4; ++a) acc[qi][a] = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      uint32_t(&cur)[32] = (c & 1) ? rb : ra;
      uint32_t(&nxt)[32] = (c & 1) ? ra : rb;
      if (c + 1 < NCH) tmem_ld_32x32b_x32(taddr0 + (c + 1) * 32, nxt);
      const int qi = c >> 1;
#pragma unroll
      for (int j = 0; j < 32; j += 4) {
        const int h = (c & 1) * 32 + j;
        const float4 wv = *reinterpret_cast<const float4*>(&wq[qi][h]);
        const float r0 = __saturatef(__uint_as_float(cur[j + 0]) * 0x1p-25f);
        const float r1 = __saturatef(__uint_as_float(cur[j + 1]) * 0x1p-25f);
        const float r2 = __saturatef(__uint_as_float(cur[j + 2]) * 0x1p-25f);
        const float r3 = __saturatef(__uint_as_float(cur[j + 3]) * 0x1p-25f);
        const int a = QPW >= 4 ? ((j >> 2) & 1) * 2 : 0;  // fewer chains when registers are scarce
        acc[qi][a] = __ffma2_rn(make_float2(wv.x, wv.y), make_float2(r0, r1), acc[qi][a]);
        acc[qi][a + 1] = __ffma2_rn(make_float2(wv.z, wv.w), make_float2(r2, r3), acc[qi][a + 1]);
      }
      if (c + 1 < NCH) tmem_wait_ld_regs(nxt);
    }
#pragma unroll
    for (int qi = 0; qi < QPW; ++qi)
      out[qi] = ((acc[qi][0].x + acc[qi][0].y) + (acc[qi][1].x + acc[qi][1].y)) +
                ((acc[qi][2].x + acc[qi][2].y) + (acc[qi][3].x + acc[qi][3].y));
  } else {
    // 8 heads per query: one scalar chain per query, four queries per chunk.
#pragma unroll
    for (int qi = 0; qi < QPW; ++qi) out[qi] = 0.0f;
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      uint32_t(&cur)[32] = (c & 1) ? rb : ra;
      uint32_t(&nxt)[32] = (c & 1) ? ra : rb;
      if (c + 1 < NCH) tmem_ld_32x32b_x32(taddr0 + (c + 1) * 32, nxt);
#pragma unroll
      for (int j = 0; j < 32; j += 4) {
        const int col = c * 32 + j;
        const int qi = col / H, h = col % H;
        const float4 wv = *reinterpret_cast<const float4*>(&wq[qi][h]);
        out[qi] = fmaf(wv.x, __saturatef(__uint_as_float(cur[j + 0]) * 0x1p-25f), out[qi]);
        out[qi] = fmaf(wv.y, __saturatef(__uint_as_float(cur[j + 1]) * 0x1p-25f), out[qi]);
        out[qi] = fmaf(wv.z, __saturatef(__uint_as_float(cur[j + 2]) * 0x1p-25f), out[qi]);
        out[qi] = fmaf(wv.w, __saturatef(__uint_as_float(cur[j + 3]) * 0x1p-25f), out[qi]);
      }
      if (c + 1 < NCH) tmem_wait_ld_regs(nxt);
    }
  }
}

// Sample and lean passes, H = 64, two queries per accumulator: the head sums read with the 16x256b TMEM
// shape. Thread t = 4g + i of the warp holds, of its lane quarter, lanes g, g+8, g+16, g+24
// (lane slot ls = lane / 8) and of each query the 16 heads 8m+2i, 8m+2i+1 (m = 0..7), so it needs
// only those 32 head weights per tile instead of all 128: the weights' broadcast loads, which
// kept the load/store unit's register writeback about three quarters busy in the 32x32b form,
// shrink fourfold. wq holds each query's weights
// permuted to [i][m][2] (wq[q][16 i + 2 m + e] = w'[q][8 m + 2 i + e]), so a thread's eight
// weights of a 32-column half are two 16-byte loads, reused for both lane halves. Returns in s
// the thread's partial sums: s[ls][q] over its 16 heads of query q.
__device__ __forceinline__ void lean_partials(uint32_t taddr0, const float* wq, uint32_t i,
                                              float (&s)[4][2]) {
  float2 acc[4][2];
#pragma unroll
  for (int ls = 0; ls < 4; ++ls)
#pragma unroll
    for (int q = 0; q < 2; ++q) acc[ls][q] = make_float2(0.0f, 0.0f);
  // Eight loads of 16 lanes x 32 columns, step k = 4 q + 2 cc + h: query q, column half cc,
  // lane half h (h fastest, so a weight octet serves two loads).
  auto addr = [&](int k) {
    return taddr0 + (static_cast<uint32_t>((k & 1) * 16) << 16) + (k >> 2) * 64 + ((k >> 1) & 1) * 32;
  };
  uint32_t ra[16], rb[16];
  float wv[8];
  tmem_ld_16x256b_x4(addr(0), ra);
  tmem_wait_ld_regs16(ra);
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    uint32_t(&cur)[16] = (k & 1) ? rb : ra;
    uint32_t(&nxt)[16] = (k & 1) ? ra : rb;
    if (k + 1 < 8) tmem_ld_16x256b_x4(addr(k + 1), nxt);
    const int q = k >> 2, cc = (k >> 1) & 1, h = k & 1;
    if (h == 0) {
      const float4 w0 = *reinterpret_cast<const float4*>(wq + q * 64 + i * 16 + cc * 8);
      const float4 w1 = *reinterpret_cast<const float4*>(wq + q * 64 + i * 16 + cc * 8 + 4);
      wv[0] = w0.x; wv[1] = w0.y; wv[2] = w0.z; wv[3] = w0.w;
      wv[4] = w1.x; wv[5] = w1.y; wv[6] = w1.z; wv[7] = w1.w;
    }
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const float2 w = make_float2(wv[2 * m], wv[2 * m + 1]);
      const float r0 = __saturatef(__uint_as_float(cur[4 * m + 0]) * 0x1p-25f);
      const float r1 = __saturatef(__uint_as_float(cur[4 * m + 1]) * 0x1p-25f);
      const float r2 = __saturatef(__uint_as_float(cur[4 * m + 2]) * 0x1p-25f);
      const float r3 = __saturatef(__uint_as_float(cur[4 * m + 3]) * 0x1p-25f);
      acc[2 * h][q] = __ffma2_rn(w, make_float2(r0, r1), acc[2 * h][q]);
      acc[2 * h + 1][q] = __ffma2_rn(w, make_float2(r2, r3), acc[2 * h + 1][q]);
    }
    if (k + 1 < 8) tmem_wait_ld_regs16(nxt);
  }
#pragma unroll
  for (int ls = 0; ls < 4; ++ls)
#pragma unroll
    for (int q = 0; q < 2; ++q) s[ls][q] = acc[ls][q].x + acc[ls][q].y;
}

// Sum of the four partials of lane slot i over the four threads 4g..4g+3 (reduce-scatter over
// xor partners 2 and 1): returns, in every thread, the full sum of its own lane slot i.
__device__ __forceinline__ float slot_total(const float (&s)[4], uint32_t i) {
  const bool hi = (i & 2u) != 0, lo = (i & 1u) != 0;
  const float send_a = hi ? s[0] : s[2], send_b = hi ? s[1] : s[3];
  const float keep_a = hi ? s[2] : s[0], keep_b = hi ? s[3] : s[1];
  const float u0 = keep_a + __shfl_xor_sync(0xFFFFFFFFu, send_a, 2);
  const float u1 = keep_b + __shfl_xor_sync(0xFFFFFFFFu, send_b, 2);
  const float send = lo ? u0 : u1, keep = lo ? u1 : u0;
  return keep + __shfl_xor_sync(0xFFFFFFFFu, send, 1);
}

template <int H, int D, int MODE>
__global__ void __launch_bounds__(PRoles<H, MODE>::THREADS, 1)
    prefill_indexer_kernel(const __grid_constant__ CUtensorMap tmap_q,
                           const __grid_constant__ CUtensorMap tmap_k, const PrefillParams p) {
  using C = PCfg<H, D>;
  extern __shared__ uint8_t smem_raw[];
  PSmem<H, D>& sm = *reinterpret_cast<PSmem<H, D>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t warp = threadIdx.x >> 5, lane = threadIdx.x & 31u;

  // Blocks this launch processes: every block, or (exact mode after a lean pass) the listed ones.
  const bool listed = MODE == kModeExact && p.fail_list != nullptr;
  const int nblocks = listed ? static_cast<int>(__ldcg(p.fail_count)) : p.nqb;
  if (nblocks <= static_cast<int>(blockIdx.x)) return;  // no block for this CTA; nothing armed yet

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&sm.kfull[s], 1);
      mbar_init(&sm.kempty[s], 1);
    }
    mbar_init(&sm.qfull, 1);
    mbar_init(&sm.qempty, 1);
    for (int g = 0; g < PRoles<H, MODE>::NACC; ++g) {
      mbar_init(&sm.accfull[g], 1);
      mbar_init(&sm.accempty[g], 4);
    }
    mbar_init(&sm.drain, 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const WaitCtl ctl{p.hdr, &sm.abort, p.budget_ns};
  const int G = gridDim.x, cta = blockIdx.x;

  // Heaviest query block first; snake order over CTAs balances the causal triangle.
  auto block_of = [&](int r) -> int {
    const int j = r * G + ((r & 1) ? (G - 1 - cta) : cta);
    if (j >= nblocks) return -1;
    return listed ? __ldcg(p.fail_list + j) : p.nqb - 1 - j;
  };
  auto ntiles_of = [&](int qb) -> int {
    const int last_t = p.q_pos0 + min(qb * C::QB + C::QB, p.Lq) - 1;
    const int last_key = min(last_t / p.stride, p.nkeys - 1);
    return last_key / C::BN + 1;
  };

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmap_q);
      prefetch_tmap(&tmap_k);
      uint32_t gi = 0, it = 0, q_issued = 0;
      uint32_t issued[C::STAGES];
      for (int s = 0; s < C::STAGES; ++s) issued[s] = 0;
      bool ok = true;
      for (int r = 0; ok; ++r) {
        const int qb = block_of(r);
        if (qb < 0) break;
        if (!mbar_wait(&sm.qempty, (it & 1u) ^ 1u, ctl, DETAIL_WAIT_QEMPTY)) break;
        mbar_arrive_expect_tx(&sm.qfull, 2 * C::QTILE);
        const int row0 = qb * C::QB * H;
        tma_load_2d(sm.q[0], &tmap_q, 0, row0, &sm.qfull);
        tma_load_2d(sm.q[1], &tmap_q, 0, row0 + 256, &sm.qfull);
        ++q_issued;
        ++it;
        const int nt = ntiles_of(qb);
        for (int tile = 0; tile < nt; ++tile, ++gi) {
          const uint32_t st = gi % C::STAGES, ph = (gi / C::STAGES) & 1u;
          if (!mbar_wait(&sm.kempty[st], ph ^ 1u, ctl, DETAIL_WAIT_KEMPTY)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&sm.kfull[st], C::KTILE);
          tma_load_2d(sm.k[st], &tmap_k, 0, tile * C::BN, &sm.kfull[st]);
          ++issued[st];
        }
      }
      // Every load this thread issued must land before the CTA can exit.
      for (int s = 0; s < C::STAGES; ++s)
        if (issued[s]) mbar_wait_drain(&sm.kfull[s], (issued[s] - 1) & 1u, p.budget_ns);
      if (q_issued) mbar_wait_drain(&sm.qfull, (q_issued - 1) & 1u, p.budget_ns);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      using R = PRoles<H, MODE>;
      uint32_t gi = 0, it = 0;
      uint32_t uses[R::NACC];
      for (int g = 0; g < R::NACC; ++g) uses[g] = 0;
      const uint32_t qa0 = smem_u32(sm.q[0]);  // the block's Q rows, R::N rows per accumulator
      bool ok = true;
      for (int r = 0; ok; ++r) {
        const int qb = block_of(r);
        if (qb < 0) break;
        if (!mbar_wait(&sm.qfull, it & 1u, ctl, DETAIL_WAIT_QFULL)) break;
        tc_fence_after();
        const int nt = ntiles_of(qb);
        for (int tile = 0; tile < nt && ok; ++tile, ++gi) {
          const uint32_t st = gi % C::STAGES, ph = (gi / C::STAGES) & 1u;
          if (!mbar_wait(&sm.kfull[st], ph, ctl, DETAIL_WAIT_KFULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t ka = smem_u32(sm.k[st]);
#pragma unroll
          for (int g = 0; g < R::NACC; ++g) {
            if (!mbar_wait(&sm.accempty[g], (uses[g] & 1u) ^ 1u, ctl, DETAIL_WAIT_ACCEMPTY)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t qa = qa0 + g * (R::N * D);
#pragma unroll
            for (int kk = 0; kk < C::KSTEPS; ++kk) {
              tc_mma_f8(tmem + g * R::N, make_smem_desc(ka + kk * 32, D),
                        make_smem_desc(qa + kk * 32, D), R::IDESC, kk > 0 ? 1u : 0u);
            }
            tc_commit(&sm.accfull[g]);
            ++uses[g];
          }
          if (ok) tc_commit(&sm.kempty[st]);
        }
        if (!ok) break;
        tc_commit(&sm.qempty);
        ++it;
      }
      // All MMAs this thread issued complete before TMEM is released.
      tc_commit(&sm.drain);
      mbar_wait_drain(&sm.drain, 0, p.budget_ns);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------------ epilogue
    using R = PRoles<H, MODE>;
    constexpr int QPW = R::QPW;
    const uint32_t g = (warp - 4) >> 2;             // accumulator (and its query group)
    const uint32_t sub = g;
    const uint32_t wl = warp & 3u;                  // TMEM lane quarter = buffer segment
    const uint32_t rank = wl * 32u + lane;          // rank within the group's 128 threads
    const GroupSync<128> gs{1u + sub};
    const uint32_t taddr0 = tmem + g * R::N + ((wl * 32u) << 16);
    const int qbase = static_cast<int>(g) * QPW;
    const uint32_t k = static_cast<uint32_t>(p.topk);
    const uint32_t segcap = p.segcap;
    const size_t pitch = 4u * static_cast<size_t>(p.seg_stride);
    const uint32_t trigger = segcap - 32u;  // exact: above it the next tile could overflow
    const uint32_t lt = (1u << lane) - 1u;
    if constexpr (MODE == kModeExact) {
      for (int i = rank; i < kHistBins; i += 128) sm.cut[sub].hist[i] = 0u;  // the selects keep it zero
    }
    uint32_t use = 0;
    bool ok = true;
    for (int r = 0; ok; ++r) {
      const int qb = block_of(r);
      if (qb < 0) break;
      const int row_base = qb * C::QB + qbase;
      for (int i = rank; i < QPW * H; i += 128) {
        const int qi = i / H, j = i % H, row = row_base + qi;
        // the sample and lean passes with H = 64 read their weights permuted (see lean_partials)
        const int slot = (MODE != kModeExact && H == 64) ? ((j & 7) >> 1) * 16 + (j >> 3) * 2 + (j & 1) : j;
        sm.wq[qbase + qi][slot] = (row < p.Lq) ? __ldg(&p.w[static_cast<size_t>(row) * H + j]) * 0x1p25f
                                               : 0.0f;
      }
      for (int qi = rank; qi < QPW; qi += 128) {
        const int row = row_base + qi;
        sm.sq[qbase + qi] = (row < p.Lq) ? __ldg(&p.q_scale[row]) : 0.0f;
        sm.thr[qbase + qi] = (MODE == kModeLean && row < p.Lq) ? __ldcg(p.thr + row) : 0ull;
      }
      if (rank == 0) sm.cflag[sub] = 0u;
      gs.sync();
      uint32_t cw[QPW];  // keys in this warp's segment, per query (warp-uniform)
#pragma unroll
      for (int qi = 0; qi < QPW; ++qi) cw[qi] = 0u;
      const int nt = ntiles_of(qb);
      // This thread's key (row of the key tensor map): its TMEM lane, or in the sample and lean
      // passes with H = 64 the lane slot the head-sum reduction leaves with it (lane g + 8 i,
      // t = 4 g + i).
      const uint32_t key_lane = (MODE != kModeExact && H == 64) ? (lane >> 2) + 8u * (lane & 3u) : lane;
      int v = static_cast<int>(wl * 32u + key_lane);
      auto scale_of = [&](int vi) {
        return vi < p.nkeys ? __ldg(&p.k_scale[static_cast<size_t>(vi) * p.stride]) : 0.0f;
      };
      float sk_next = scale_of(v);
      bool good = true;
      if constexpr (MODE != kModeExact && H == 64) {
        // Per query of this warp, in registers: the threshold T as (score, largest key index
        // taken at that score) and the query scale; the queries' segments are one row pitch
        // apart. key >= T  <=>  score > score(T), or score == score(T) and s <= index(T).
        float tf[QPW], sqr[QPW];
        uint32_t tix[QPW];
#pragma unroll
        for (int qi = 0; qi < QPW; ++qi) {
          const uint64_t T = sm.thr[qbase + qi];
          tf[qi] = key_score(T);  // -inf for T = 0: every key is taken
          tix[qi] = T ? static_cast<uint32_t>(key_index(T)) : 0xFFFFFFFFu;
          sqr[qi] = sm.sq[qbase + qi];
        }
        uint64_t* const dst0 = p.cand + static_cast<size_t>(row_base) * pitch + wl * p.seg_stride;
        // Tiles whose keys all lie at or before the earlier query's position need no mask
        // (every such key is also below Lk); only the diagonal tiles are masked. The sample pass
        // reads every S-th key (map row v is key S v) and appends every valid one (T = 0).
        const bool rows_ok = row_base + QPW - 1 < p.Lq;
        const int n_plain = rows_ok ? min(nt, ((p.q_pos0 + row_base) / p.stride + 1) / C::BN) : 0;
        auto lean_tile = [&](auto masked_tag) {
          constexpr bool MASKED = decltype(masked_tag)::value;
          const float sk = sk_next;
          sk_next = __ldg(&p.k_scale[static_cast<size_t>(min(v + C::BN, p.nkeys - 1)) * p.stride]);
          const int s = v * p.stride;  // the key's position
          const bool got = mbar_wait(&sm.accfull[g], use & 1u, ctl, DETAIL_WAIT_ACCFULL);
          good = good && got;
          __syncwarp();
          tc_fence_after();
          float part[4][2];
          lean_partials(taddr0, &sm.wq[qbase][0], lane & 3u, part);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.accempty[g]);
          ++use;
          float score_part[QPW];
#pragma unroll
          for (int qi = 0; qi < QPW; ++qi) {
            const float col[4] = {part[0][qi], part[1][qi], part[2][qi], part[3][qi]};
            score_part[qi] = slot_total(col, lane & 3u);
          }
#pragma unroll
          for (int qi = 0; qi < QPW; ++qi) {
            const float score = (score_part[qi] * sqr[qi]) * sk;
            bool take = score > tf[qi] || (score == tf[qi] && static_cast<uint32_t>(s) <= tix[qi]);
            if constexpr (MASKED) take = take && (row_base + qi < p.Lq) && (s <= p.q_pos0 + row_base + qi);
            const uint32_t m = __ballot_sync(0xFFFFFFFFu, take);
            if (m) {  // warp-uniform: most warps of a long row append nothing
              const uint32_t pos = cw[qi] + __popc(m & lt);
              if (take && pos < segcap) dst0[qi * pitch + pos] = make_key(score, static_cast<uint32_t>(s));
              cw[qi] += __popc(m);
            }
          }
          v += C::BN;
        };
        int tile = 0;
        for (; tile < n_plain; ++tile) lean_tile(std::integral_constant<bool, false>{});
        for (; tile < nt; ++tile) lean_tile(std::integral_constant<bool, true>{});
      } else {
      for (int tile = 0; tile < nt; ++tile, v += C::BN) {
        const float sk = sk_next;
        sk_next = scale_of(v + C::BN);
        const int s = v * p.stride;  // the key's position
        const bool got = mbar_wait(&sm.accfull[g], use & 1u, ctl, DETAIL_WAIT_ACCFULL);
        good = good && got;
        __syncwarp();
        tc_fence_after();
        float score_part[QPW];
        head_sums<H, QPW>(taddr0, &sm.wq[qbase], score_part);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.accempty[g]);
        ++use;

        // Appends to this warp's own segment: no atomics, the count lives in a register.
        uint32_t flags = 0u;
#pragma unroll
        for (int qi = 0; qi < QPW; ++qi) {
          const int row = row_base + qi;
          const bool valid = (row < p.Lq) && (v < p.nkeys) && (s <= p.q_pos0 + row);
          const float score = (score_part[qi] * sm.sq[qbase + qi]) * sk;
          const uint64_t key = make_key(score, static_cast<uint32_t>(s));
          const bool take = valid && (MODE == kModeSample || key >= sm.thr[qbase + qi]);
          const uint32_t m = __ballot_sync(0xFFFFFFFFu, take);
          const uint32_t pos = cw[qi] + __popc(m & lt);
          if (take && pos < segcap) p.cand[static_cast<size_t>(row) * pitch + wl * p.seg_stride + pos] = key;
          cw[qi] += __popc(m);
          if constexpr (MODE == kModeExact) flags |= (cw[qi] > trigger) ? (1u << qi) : 0u;
        }
        if constexpr (MODE == kModeExact) {
          // Cut-backs: one decision for the whole group. The barrier ORs the warps' requests,
          // and the flag word written before it is visible to every warp after it.
          if (flags && lane == 0) atomicOr(&sm.cflag[sub], flags);
          if (named_bar_or(1u + sub, 128, flags != 0u)) {
            const uint32_t mask = *reinterpret_cast<volatile uint32_t*>(&sm.cflag[sub]);
            if (lane == 0) {
#pragma unroll
              for (int qi = 0; qi < QPW; ++qi) sm.wcnt[qbase + qi][wl] = cw[qi];
            }
            gs.sync();
            if (rank == 0) sm.cflag[sub] = 0u;
#pragma unroll 1
            for (int qi = 0; qi < QPW; ++qi) {
              if ((mask >> qi) & 1u)
                cut_back(p.cand + static_cast<size_t>(row_base + qi) * pitch, p.seg_stride,
                         sm.wcnt[qbase + qi], &sm.thr[qbase + qi], &sm.cut[sub], k, rank, 1u + sub);
            }
#pragma unroll
            for (int qi = 0; qi < QPW; ++qi) cw[qi] = sm.wcnt[qbase + qi][wl];
          }
        }
      }
      }
      ok = named_bar_and(1u + sub, 128, ok && good);
      if (!ok) break;
      // Segment counts (and thresholds) of every query of this group.
      if (lane == 0) {
#pragma unroll
        for (int qi = 0; qi < QPW; ++qi) {
          const int row = row_base + qi;
          if (row < p.Lq) p.counts[static_cast<size_t>(row) * 4 + wl] = cw[qi];
          sm.wcnt[qbase + qi][wl] = cw[qi];
        }
      }
      if constexpr (MODE == kModeExact) {
        for (int qi = rank; qi < QPW; qi += 128) {
          const int row = row_base + qi;
          if (row < p.Lq) p.thr[row] = sm.thr[qbase + qi];
        }
      }
      if constexpr (MODE == kModeLean) {
        // A query whose buffer lacks some of its top-k (fewer than min(k, keys in its row)
        // appended), or whose segment overflowed, sends its block to the exact mode.
        gs.sync();
        bool bad = false;
        for (int qi = rank; qi < QPW; qi += 128) {
          const int row = row_base + qi;
          if (row >= p.Lq) continue;
          uint32_t total = 0;
          bool full = false;
          for (int w = 0; w < 4; ++w) {
            const uint32_t c = sm.wcnt[qbase + qi][w];
            total += c;
            full = full || c > segcap;
          }
          const uint32_t keys = static_cast<uint32_t>(min(p.q_pos0 + row + 1, p.Lk));
          bad = bad || full || total < min(k, keys);
        }
        if (bad && atomicCAS(p.fail_flag + qb, 0u, 1u) == 0u)
          p.fail_list[atomicAdd(p.fail_count, 1u)] = qb;
        gs.sync();  // wcnt is rewritten for the next block
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Key stride S of the sample pass for top-k over rows of up to Lk keys: about k / S >= 64
// sampled keys lie above a row's k-th largest key, and a row's sample (ceil(Lk / S) keys)
// fits its buffer. 1 means no sample pass: every block runs in the exact mode. The sample pass
// and the threshold cost about Lk / S per row, while the keys a row keeps above its threshold
// grow only as k + 6.5 sqrt(k S); long rows (Lk >= 24576) take twice the stride.
static int sample_stride(int topk, int Lk, uint32_t seg_stride) {
  int S = topk / 128;
  if (S < 2) return 1;
  if (Lk >= 24576) S *= 2;
  const int64_t room = 4 * static_cast<int64_t>(seg_stride) - 4 * 32;  // tiles end on 32-key boundaries
  const int min_s = static_cast<int>((static_cast<int64_t>(Lk) + room - 1) / room);
  return S > min_s ? S : min_s;
}

template <int H, int D, int MODE>
static dsa_status launch_mode(const CUtensorMap& tq, const CUtensorMap& tk, const PrefillParams& p,
                              int grid, cudaStream_t stream) {
  using C = PCfg<H, D>;
  // At least half of the SM's shared memory, so that one CTA (and its 512 TMEM columns)
  // owns each SM.
  size_t smem = sizeof(PSmem<H, D>) + 1024;
  if (smem < 120 * 1024) smem = 120 * 1024;
  auto kern = prefill_indexer_kernel<H, D, MODE>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return DSA_ERR_CUDA;
  kern<<<grid, PRoles<H, MODE>::THREADS, smem, stream>>>(tq, tk, p);
  return cuda_status(cudaGetLastError());
}

template <int H, int D>
static dsa_status launch_prefill_t(const PrefillLaunch& a) {
  using C = PCfg<H, D>;
  const PrefillLayout L = prefill_layout(a.Lq, a.topk);
  const int nqb = (a.Lq + C::QB - 1) / C::QB;
  const int grid = nqb < a.num_sms ? nqb : a.num_sms;
  uint8_t* base = static_cast<uint8_t*>(a.ws);
  PrefillParams p{};
  p.q_scale = a.q_scale;
  p.w = a.w;
  p.k_scale = a.k_scale;
  p.Lk = a.Lk;
  p.q_pos0 = a.q_pos0;
  p.Lq = a.Lq;
  p.topk = a.topk;
  p.nqb = nqb;
  p.stride = 1;
  p.nkeys = a.Lk;
  p.seg_stride = L.seg_stride;
  p.segcap = L.exact_segcap;
  p.hdr = reinterpret_cast<WsHeader*>(base);
  p.cand = reinterpret_cast<uint64_t*>(base + L.cand_off);
  p.thr = reinterpret_cast<uint64_t*>(base + L.thr_off);
  p.counts = reinterpret_cast<uint32_t*>(base + L.counts_off);
  p.fail_flag = reinterpret_cast<uint32_t*>(base + L.flags_off);
  p.fail_list = reinterpret_cast<int32_t*>(base + L.list_off);
  p.fail_count = reinterpret_cast<uint32_t*>(base + L.count_off);
  p.budget_ns = a.budget_ns;

  CUtensorMap tq, tk;
  if (!encode_tmap_2d_u8(&tq, a.q, D, static_cast<uint64_t>(a.Lq) * H, 256)) return DSA_ERR_CUDA;
  if (!encode_tmap_2d_u8(&tk, a.k, D, static_cast<uint64_t>(a.Lk), 128)) return DSA_ERR_CUDA;

  const int S = sample_stride(a.topk, a.Lk, L.seg_stride);
  dsa_status st;
  if (S > 1) {
    // Sample pass over keys 0, S, 2S, ...: every valid sampled key appended.
    CUtensorMap ts;
    const int nks = (a.Lk + S - 1) / S;
    if (!encode_tmap_2d_u8(&ts, a.k, D, static_cast<uint64_t>(nks), 128, static_cast<uint64_t>(S) * D))
      return DSA_ERR_CUDA;
    PrefillParams ps = p;
    ps.stride = S;
    ps.nkeys = nks;
    ps.segcap = L.seg_stride;
    if ((st = launch_mode<H, D, kModeSample>(tq, ts, ps, grid, a.stream)) != DSA_OK) return st;
    if ((st = launch_prefill_sample_threshold(p.cand, p.counts, p.thr, L.seg_stride, a.Lq, a.q_pos0,
                                              a.Lk, a.topk, static_cast<uint32_t>(nks), a.stream)) != DSA_OK)
      return st;
    // Lean pass with those thresholds; blocks it cannot finish are listed for the exact mode.
    if (cudaMemsetAsync(base + L.flags_off, 0, L.total - L.flags_off, a.stream) != cudaSuccess)
      return DSA_ERR_CUDA;
    PrefillParams pl = p;
    pl.segcap = L.lean_segcap;
    if ((st = launch_mode<H, D, kModeLean>(tq, tk, pl, grid, a.stream)) != DSA_OK) return st;
    if ((st = launch_mode<H, D, kModeExact>(tq, tk, p, grid, a.stream)) != DSA_OK) return st;
  } else {
    PrefillParams pe = p;
    pe.fail_list = nullptr;
    if ((st = launch_mode<H, D, kModeExact>(tq, tk, pe, grid, a.stream)) != DSA_OK) return st;
  }
  return launch_prefill_finish(p.cand, p.counts, p.thr, 4u * L.seg_stride, a.Lq, a.topk,
                               a.out_idx, a.out_score, a.num_sms, a.stream);
}

size_t prefill_workspace_bytes(int Lq, int H, int d, int topk, int num_sms) {
  (void)H;
  (void)d;
  (void)num_sms;
  return prefill_layout(Lq, topk).total;
}

dsa_status launch_prefill(const PrefillLaunch& a) {
  if (a.H == 64 && a.d == 128) return launch_prefill_t<64, 128>(a);
  if (a.H == 8 && a.d == 64) return launch_prefill_t<8, 64>(a);
  return DSA_ERR_UNSUPPORTED;
}

}  // namespace dsa

// Fused prefill lightning indexer for sm_100a.
//
// One persistent CTA per SM walks query blocks (heaviest first, snake order over CTAs).
// For a block of QB queries it streams the causal key range in tiles of 128 keys:
//   warp 0      TMA producer: the block's Q rows (two 256-row B operands) once, then one
//               [128 keys x d] FP8 K tile per pipeline stage;
//   warp 1      one thread issues tcgen05.mma kind::f8f6f4 (M = 128 keys, N = 256 =
//               (256/H) queries x H heads, K = d), FP32 accumulators in TMEM, two
//               256-column accumulators so the epilogue of one overlaps the MMA of the other;
//   warps 4-11  two epilogue warpgroups, one per accumulator. Thread = key (its TMEM lane):
//               it reads the key's H head dot products of each query, applies
//               ReLU, the head weights, then the query and key scales, masks s > t, and
//               streams keys that can still enter the top-k into a per-query candidate
//               buffer (workspace). A nearly full buffer is staged in shared memory and cut
//               back to exactly topk keys by an exact radix select, which also raises the
//               query's insertion threshold.
// After the last tile every query's buffer is reduced to exactly its top-k keys and written
// to the winners array; the row sort (topk.cu) orders them. The L x L score matrix is never
// stored.
//
// ReLU on the FMA pipe: D = q8.k8 with |D| <= d * 448^2 < 2^25, so
// max(D, 0) = 2^25 * sat(D * 2^-25) exactly (power-of-two scalings, no clipping at 1), and
// the 2^25 is folded into the stored head weights.
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
  static constexpr int THREADS = 384;
  static constexpr int NP = (H >= 32) ? 4 : 1;  // partial sums per query (ILP)
  static constexpr uint32_t IDESC = make_idesc_f8(128, 256);
  static_assert(D == 64 || D == 128, "d");
  static_assert(H == 8 || H == 64, "H");
};

constexpr int kCandCapMax = 2 * DSA_MAX_TOPK + 256;

template <int H, int D>
struct PSmem {
  using C = PCfg<H, D>;
  uint8_t q[2][C::QTILE];
  uint8_t k[C::STAGES][C::KTILE];
  float wq[C::QB][H];
  float sq[C::QB];
  uint64_t thr[C::QB];
  uint32_t cnt[C::QB];
  uint32_t hist[2][kHistBins];
  GroupScratch<128> gsc[2];
  uint64_t stage[2][kCandCapMax];   // a candidate buffer staged for a cut-back
  uint64_t kfull[C::STAGES];
  uint64_t kempty[C::STAGES];
  uint64_t qfull, qempty, accfull[2], accempty[2], drain;
  uint32_t tmem_base;
  int abort;
};

// Copies n candidate keys from global memory into shared memory, eight independent loads in
// flight per thread.
__device__ __forceinline__ void stage_keys(const uint64_t* __restrict__ src, uint32_t n,
                                           uint64_t* __restrict__ dst, uint32_t rank) {
  uint32_t e = rank;
  for (; e + 7 * 128 < n; e += 8 * 128) {
    uint64_t v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __ldcg(src + e + i * 128);
#pragma unroll
    for (int i = 0; i < 8; ++i) dst[e + i * 128] = v[i];
  }
  for (; e < n; e += 128) dst[e] = __ldcg(src + e);
}

struct PrefillParams {
  const float* q_scale;
  const float* w;
  const float* k_scale;
  int32_t Lk, q_pos0, Lq, topk;
  int32_t nqb;
  uint32_t cap;
  uint64_t* cand;
  uint64_t* win;
  WsHeader* hdr;
  uint64_t budget_ns;
};

template <int H, int D>
__global__ void __launch_bounds__(384, 1)
    prefill_indexer_kernel(const __grid_constant__ CUtensorMap tmap_q,
                           const __grid_constant__ CUtensorMap tmap_k, const PrefillParams p) {
  using C = PCfg<H, D>;
  extern __shared__ uint8_t smem_raw[];
  PSmem<H, D>& sm = *reinterpret_cast<PSmem<H, D>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t warp = threadIdx.x >> 5, lane = threadIdx.x & 31u;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&sm.kfull[s], 1);
      mbar_init(&sm.kempty[s], 1);
    }
    mbar_init(&sm.qfull, 1);
    mbar_init(&sm.qempty, 1);
    for (int g = 0; g < 2; ++g) {
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
    return j < p.nqb ? p.nqb - 1 - j : -1;
  };
  auto ntiles_of = [&](int qb) -> int {
    const int last_row = min(qb * C::QB + C::QB, p.Lq) - 1;
    return (p.q_pos0 + last_row) / C::BN + 1;
  };
  auto cand_buf = [&](int qidx) -> uint64_t* {
    return p.cand + (static_cast<size_t>(cta) * C::QB + qidx) * p.cap;
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
      uint32_t gi = 0, it = 0, use0 = 0, use1 = 0;
      const uint32_t qa0 = smem_u32(sm.q[0]), qa1 = smem_u32(sm.q[1]);
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
          for (int g = 0; g < 2; ++g) {
            const uint32_t use = g ? use1 : use0;
            if (!mbar_wait(&sm.accempty[g], (use & 1u) ^ 1u, ctl, DETAIL_WAIT_ACCEMPTY)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t qa = g ? qa1 : qa0;
#pragma unroll
            for (int kk = 0; kk < C::KSTEPS; ++kk) {
              tc_mma_f8(tmem + g * 256, make_smem_desc(ka + kk * 32, D),
                        make_smem_desc(qa + kk * 32, D), C::IDESC, kk > 0 ? 1u : 0u);
            }
            tc_commit(&sm.accfull[g]);
            if (g) ++use1; else ++use0;
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
    const uint32_t g = (warp - 4) >> 2;       // accumulator / warpgroup
    const uint32_t wl = warp & 3u;            // TMEM lane quarter of this warp
    const uint32_t rank = threadIdx.x - 128u * (1u + g);
    const GroupSync<128> gs{1u + g};
    uint32_t* hist = sm.hist[g];
    GroupScratch<128>& scr = sm.gsc[g];
    uint64_t* stage = sm.stage[g];
    const uint32_t taddr0 = tmem + g * 256 + ((wl * 32u) << 16);
    const int qbase = static_cast<int>(g) * C::QPM;
    uint32_t use = 0;
    bool ok = true;
    for (int r = 0; ok; ++r) {
      const int qb = block_of(r);
      if (qb < 0) break;
      const int row_base = qb * C::QB + qbase;
      for (int e = rank; e < C::QPM * H; e += 128) {
        const int qi = e / H, j = e % H, row = row_base + qi;
        sm.wq[qbase + qi][j] = (row < p.Lq) ? __ldg(&p.w[static_cast<size_t>(row) * H + j]) * 0x1p25f
                                            : 0.0f;
      }
      for (int qi = rank; qi < C::QPM; qi += 128) {
        const int row = row_base + qi;
        sm.sq[qbase + qi] = (row < p.Lq) ? __ldg(&p.q_scale[row]) : 0.0f;
        sm.thr[qbase + qi] = 0;
        sm.cnt[qbase + qi] = 0;
      }
      gs.sync();
      const int nt = ntiles_of(qb);
      for (int tile = 0; tile < nt; ++tile) {
        const int s = tile * C::BN + static_cast<int>(wl * 32u + lane);
        const float sk = (s < p.Lk) ? __ldg(&p.k_scale[s]) : 0.0f;
        const bool got = mbar_wait(&sm.accfull[g], use & 1u, ctl, DETAIL_WAIT_ACCFULL);
        __syncwarp();
        tc_fence_after();
        float part[C::QPM][C::NP];
#pragma unroll
        for (int qi = 0; qi < C::QPM; ++qi)
#pragma unroll
          for (int pp = 0; pp < C::NP; ++pp) part[qi][pp] = 0.0f;
        uint32_t ra[32], rb[32];
        tmem_ld_32x32b_x32(taddr0, ra);
        tmem_wait_ld_regs(ra);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t(&cur)[32] = (c & 1) ? rb : ra;
          uint32_t(&nxt)[32] = (c & 1) ? ra : rb;
          if (c + 1 < 8) tmem_ld_32x32b_x32(taddr0 + (c + 1) * 32, nxt);
#pragma unroll
          for (int j = 0; j < 32; j += 4) {
            const int col = c * 32 + j;
            const int qi = col / H, h = col % H;
            const float4 wv = *reinterpret_cast<const float4*>(&sm.wq[qbase + qi][h]);
            part[qi][(j + 0) % C::NP] = fmaf(wv.x, __saturatef(__uint_as_float(cur[j + 0]) * 0x1p-25f), part[qi][(j + 0) % C::NP]);
            part[qi][(j + 1) % C::NP] = fmaf(wv.y, __saturatef(__uint_as_float(cur[j + 1]) * 0x1p-25f), part[qi][(j + 1) % C::NP]);
            part[qi][(j + 2) % C::NP] = fmaf(wv.z, __saturatef(__uint_as_float(cur[j + 2]) * 0x1p-25f), part[qi][(j + 2) % C::NP]);
            part[qi][(j + 3) % C::NP] = fmaf(wv.w, __saturatef(__uint_as_float(cur[j + 3]) * 0x1p-25f), part[qi][(j + 3) % C::NP]);
          }
          if (c + 1 < 8) tmem_wait_ld_regs(nxt);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.accempty[g]);
        ++use;

#pragma unroll
        for (int qi = 0; qi < C::QPM; ++qi) {
          float acc = part[qi][0];
#pragma unroll
          for (int pp = 1; pp < C::NP; ++pp) acc += part[qi][pp];
          const int row = row_base + qi;
          const bool valid = (row < p.Lq) && (s <= p.q_pos0 + row);
          const float score = (acc * sm.sq[qbase + qi]) * sk;
          const uint64_t key = make_key(score, static_cast<uint32_t>(s));
          const bool take = valid && key >= sm.thr[qbase + qi];
          const uint32_t m = __ballot_sync(0xFFFFFFFFu, take);
          if (m) {
            uint32_t base = 0;
            if (lane == 0) base = atomicAdd(&sm.cnt[qbase + qi], static_cast<uint32_t>(__popc(m)));
            base = __shfl_sync(0xFFFFFFFFu, base, 0);
            if (take) cand_buf(qbase + qi)[base + __popc(m & ((1u << lane) - 1u))] = key;
          }
        }
        ok = named_bar_and(1u + g, 128, ok && got);
        if (!ok) break;
        // Cut any nearly full candidate buffer back to exactly topk keys: stage it in shared
        // memory, find the threshold there, write the survivors back to the buffer's front.
        for (int qi = 0; qi < C::QPM; ++qi) {
          const uint32_t n = sm.cnt[qbase + qi];
          if (n <= p.cap - 128u) continue;
          uint64_t* buf = cand_buf(qbase + qi);
          stage_keys(buf, n, stage, rank);
          gs.sync();
          auto key_at = [&](uint32_t e) { return stage[e]; };
          const uint32_t k = static_cast<uint32_t>(p.topk);
          const uint64_t T = group_kth_threshold<128>(key_at, n, k, rank, hist, scr, gs);
          group_compact_ge<128>(key_at, n, T,
                                [&](uint32_t pos, uint64_t key) { if (pos < k) buf[pos] = key; },
                                rank, scr, gs);
          if (rank == 0) {
            sm.thr[qbase + qi] = T;
            sm.cnt[qbase + qi] = k;
          }
          gs.sync();
        }
      }
      if (!ok) break;
      // Final top-k of every query of this warpgroup -> winners[row][0..topk).
      for (int qi = 0; qi < C::QPM; ++qi) {
        const int row = row_base + qi;
        if (row >= p.Lq) break;
        const uint32_t n = sm.cnt[qbase + qi];
        const uint32_t k = static_cast<uint32_t>(p.topk);
        const uint64_t* buf = cand_buf(qbase + qi);
        uint64_t* dst = p.win + static_cast<size_t>(row) * p.topk;
        if (n > k) {
          stage_keys(buf, n, stage, rank);
          gs.sync();
          auto key_at = [&](uint32_t e) { return stage[e]; };
          const uint64_t T = group_kth_threshold<128>(key_at, n, k, rank, hist, scr, gs);
          group_compact_ge<128>(key_at, n, T,
                                [&](uint32_t pos, uint64_t key) { if (pos < k) dst[pos] = key; },
                                rank, scr, gs);
        } else {
          for (uint32_t e = rank; e < k; e += 128) dst[e] = (e < n) ? buf[e] : 0ull;
        }
        gs.sync();
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int H, int D>
static dsa_status launch_prefill_t(const PrefillLaunch& a) {
  using C = PCfg<H, D>;
  // At least half of the SM's shared memory, so that one CTA (and its 512 TMEM columns)
  // owns each SM.
  size_t smem = sizeof(PSmem<H, D>) + 1024;
  if (smem < 120 * 1024) smem = 120 * 1024;
  auto kern = prefill_indexer_kernel<H, D>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return DSA_ERR_CUDA;
  CUtensorMap tq, tk;
  if (!encode_tmap_2d_u8(&tq, a.q, D, static_cast<uint64_t>(a.Lq) * H, 256)) return DSA_ERR_CUDA;
  if (!encode_tmap_2d_u8(&tk, a.k, D, static_cast<uint64_t>(a.Lk), 128)) return DSA_ERR_CUDA;

  const int nqb = (a.Lq + C::QB - 1) / C::QB;
  const int grid = nqb < a.num_sms ? nqb : a.num_sms;
  uint8_t* base = static_cast<uint8_t*>(a.ws);
  PrefillParams p;
  p.q_scale = a.q_scale;
  p.w = a.w;
  p.k_scale = a.k_scale;
  p.Lk = a.Lk;
  p.q_pos0 = a.q_pos0;
  p.Lq = a.Lq;
  p.topk = a.topk;
  p.nqb = nqb;
  p.cap = prefill_cand_cap(a.topk);
  p.hdr = reinterpret_cast<WsHeader*>(base);
  p.cand = reinterpret_cast<uint64_t*>(base + DSA_WS_HEADER_BYTES);
  const size_t cand_bytes = static_cast<size_t>(a.num_sms) * C::QB * p.cap * sizeof(uint64_t);
  p.win = reinterpret_cast<uint64_t*>(base + DSA_WS_HEADER_BYTES + cand_bytes);
  p.budget_ns = a.budget_ns;
  kern<<<grid, C::THREADS, smem, a.stream>>>(tq, tk, p);
  if (cudaGetLastError() != cudaSuccess) return DSA_ERR_CUDA;
  return launch_sort_rows(p.win, a.Lq, a.topk, a.out_idx, a.out_score, a.stream);
}

size_t prefill_workspace_bytes(int Lq, int H, int d, int topk, int num_sms) {
  (void)d;
  const size_t qb = static_cast<size_t>(prefill_queries_per_block(H));
  const size_t cand = static_cast<size_t>(num_sms) * qb * prefill_cand_cap(topk) * sizeof(uint64_t);
  const size_t win = static_cast<size_t>(Lq) * topk * sizeof(uint64_t);
  return DSA_WS_HEADER_BYTES + cand + win;
}

dsa_status launch_prefill(const PrefillLaunch& a) {
  if (a.H == 64 && a.d == 128) return launch_prefill_t<64, 128>(a);
  if (a.H == 8 && a.d == 64) return launch_prefill_t<8, 64>(a);
  return DSA_ERR_UNSUPPORTED;
}

}  // namespace dsa

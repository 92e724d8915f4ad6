// Decode lightning indexer for sm_100a: one query (H = 64 heads) per request against its
// paged FP8 key cache.
//
// Grid (chunks, B): CTA (c, b) scores tiles [c*TPC, (c+1)*TPC) of request b, a tile being 128
// logical keys = two 64-key pages. The work is HBM-bound (d + 4 bytes per key), so the CTA is
// small (three fit per SM) and keeps STAGES tiles in flight:
//   warp 0     TMA: the request's 64 query rows once, then per tile the two pages named by
//              the block table (entries are range-checked; a bad entry is recorded as
//              DSA_ERR_DEVICE and block 0 is read instead);
//   warp 1     one thread issues tcgen05.mma kind::f8f6f4, M = 128 keys, N = 64 heads,
//              K = d, into one of two 64-column TMEM accumulators;
//   warps 2-5  epilogue: thread = key; ReLU (on the FMA pipe, see prefill.cu), head weights,
//              scales; the score of every valid key is stored at scores[b][s] and counted in
//              the request's histogram of order-preserving top-11-bit bins.
// decode_topk_kernel (topk.cu) then selects and orders each request's top-k.
#include "common.cuh"
#include "internal.h"

namespace dsa {

constexpr int kScoreBins = kDecodeScoreBins;  // bins of the top 11 bits of an order-preserving fp32 key

template <int D>
struct DCfg {
  static constexpr int H = 64;
  static constexpr int PAGE = 64;              // keys per cache block
  static constexpr int BN = 128;               // keys per tile
  static constexpr int STAGES = 3;
  static constexpr int TPC = 16;               // tiles per CTA
  static constexpr int QTILE = H * D;
  static constexpr int KTILE = BN * D;
  static constexpr int PAGE_BYTES = PAGE * D;
  static constexpr int KSTEPS = D / 32;
  static constexpr int THREADS = 192;
  static constexpr uint32_t IDESC = make_idesc_f8(128, 64);
};

template <int D>
struct DSmem {
  using C = DCfg<D>;
  uint8_t q[C::QTILE];
  uint8_t k[C::STAGES][C::KTILE];
  float wq[C::H];
  uint32_t hist[kScoreBins];   // this CTA's scores per order-preserving top-11-bit bin
  uint64_t kfull[C::STAGES];
  uint64_t kempty[C::STAGES];
  uint64_t qfull, accfull[2], accempty[2], drain;
  uint32_t tmem_base;
  int abort;
};

struct DecodeParams {
  const float* q_scale;
  const float* w;
  const float* k_scale_cache;
  const int32_t* block_table;
  const int32_t* seq_lens;
  int32_t max_blocks, n_blocks, max_len;
  float* scores;
  uint32_t* bins;   // [B][kScoreBins] per-request score histogram
  WsHeader* hdr;
  uint64_t budget_ns;
};

template <int D>
__global__ void __launch_bounds__(192)
    decode_indexer_kernel(const __grid_constant__ CUtensorMap tmap_q,
                          const __grid_constant__ CUtensorMap tmap_k, const DecodeParams p) {
  using C = DCfg<D>;
  const int b = blockIdx.y;
  int n = __ldg(&p.seq_lens[b]);
  if (n < 1 || n > p.max_len) {
    if (blockIdx.x == 0 && threadIdx.x == 0) record_error(p.hdr, DSA_ERR_DEVICE, DETAIL_BAD_SEQ_LEN);
    n = n < 1 ? 1 : p.max_len;
  }
  const int ntiles = (n + C::BN - 1) / C::BN;
  const int t0 = blockIdx.x * C::TPC;
  if (t0 >= ntiles) return;  // uniform over the CTA, before any shared state exists
  const int t1 = min(ntiles, t0 + C::TPC);
  const int nblk_req = (n + C::PAGE - 1) / C::PAGE;
  const int32_t* table = p.block_table + static_cast<size_t>(b) * p.max_blocks;

  extern __shared__ uint8_t smem_raw[];
  DSmem<D>& sm = *reinterpret_cast<DSmem<D>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t warp = threadIdx.x >> 5, lane = threadIdx.x & 31u;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&sm.kfull[s], 1);
      mbar_init(&sm.kempty[s], 1);
    }
    mbar_init(&sm.qfull, 1);
    for (int a = 0; a < 2; ++a) {
      mbar_init(&sm.accfull[a], 1);
      mbar_init(&sm.accempty[a], 4);
    }
    mbar_init(&sm.drain, 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const WaitCtl ctl{p.hdr, &sm.abort, p.budget_ns};

  auto phys_block = [&](int lb, bool record) -> int {
    int pb = __ldg(&table[lb]);
    if (pb < 0 || pb >= p.n_blocks) {
      if (record) record_error(p.hdr, DSA_ERR_DEVICE, DETAIL_BAD_BLOCK_TABLE);
      pb = 0;
    }
    return pb;
  };

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tmap_q);
      prefetch_tmap(&tmap_k);
      mbar_arrive_expect_tx(&sm.qfull, C::QTILE);
      tma_load_2d(sm.q, &tmap_q, 0, b * C::H, &sm.qfull);
      uint32_t issued[C::STAGES];
      for (int s = 0; s < C::STAGES; ++s) issued[s] = 0;
      uint32_t gi = 0;
      for (int tile = t0; tile < t1; ++tile, ++gi) {
        const uint32_t st = gi % C::STAGES, ph = (gi / C::STAGES) & 1u;
        if (!mbar_wait(&sm.kempty[st], ph ^ 1u, ctl, DETAIL_WAIT_KEMPTY)) break;
        const int lb0 = 2 * tile, lb1 = 2 * tile + 1;
        const bool two = lb1 < nblk_req;
        mbar_arrive_expect_tx(&sm.kfull[st], two ? 2 * C::PAGE_BYTES : C::PAGE_BYTES);
        tma_load_2d(sm.k[st], &tmap_k, 0, phys_block(lb0, true) * C::PAGE, &sm.kfull[st]);
        if (two)
          tma_load_2d(sm.k[st] + C::PAGE_BYTES, &tmap_k, 0, phys_block(lb1, true) * C::PAGE,
                      &sm.kfull[st]);
        ++issued[st];
      }
      for (int s = 0; s < C::STAGES; ++s)
        if (issued[s]) mbar_wait_drain(&sm.kfull[s], (issued[s] - 1) & 1u, p.budget_ns);
      mbar_wait_drain(&sm.qfull, 0, p.budget_ns);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      uint32_t use[2] = {0, 0};
      if (mbar_wait(&sm.qfull, 0, ctl, DETAIL_WAIT_QFULL)) {
        tc_fence_after();
        const uint32_t qa = smem_u32(sm.q);
        uint32_t gi = 0;
        for (int tile = t0; tile < t1; ++tile, ++gi) {
          const uint32_t st = gi % C::STAGES, ph = (gi / C::STAGES) & 1u;
          const uint32_t a = gi & 1u;
          if (!mbar_wait(&sm.kfull[st], ph, ctl, DETAIL_WAIT_KFULL)) break;
          if (!mbar_wait(&sm.accempty[a], (use[a] & 1u) ^ 1u, ctl, DETAIL_WAIT_ACCEMPTY)) break;
          tc_fence_after();
          const uint32_t ka = smem_u32(sm.k[st]);
#pragma unroll
          for (int kk = 0; kk < C::KSTEPS; ++kk)
            tc_mma_f8(tmem + a * 64, make_smem_desc(ka + kk * 32, D), make_smem_desc(qa + kk * 32, D),
                      C::IDESC, kk > 0 ? 1u : 0u);
          tc_commit(&sm.accfull[a]);
          tc_commit(&sm.kempty[st]);
          ++use[a];
        }
      }
      tc_commit(&sm.drain);
      mbar_wait_drain(&sm.drain, 0, p.budget_ns);
    }
    __syncwarp();
  } else {
    // epilogue warps 2..5 -> TMEM lane quarters 2, 3, 0, 1
    const uint32_t wl = warp & 3u;
    const uint32_t rank = threadIdx.x - 64u;
    if (rank < C::H) sm.wq[rank] = __ldg(&p.w[static_cast<size_t>(b) * C::H + rank]) * 0x1p25f;
    for (int i = rank; i < kScoreBins; i += 128) sm.hist[i] = 0u;
    named_bar(1, 128);
    const float sq = __ldg(&p.q_scale[b]);
    float* out = p.scores + static_cast<size_t>(b) * p.max_len;
    uint32_t use[2] = {0, 0};
    uint32_t gi = 0;
    for (int tile = t0; tile < t1; ++tile, ++gi) {
      const uint32_t a = gi & 1u;
      const int s = tile * C::BN + static_cast<int>(wl * 32u + lane);
      const bool valid = s < n;
      float sk = 0.0f;
      if (valid) {
        const int pb = phys_block(s / C::PAGE, false);
        sk = __ldg(&p.k_scale_cache[static_cast<size_t>(pb) * C::PAGE + (s % C::PAGE)]);
      }
      const bool got = mbar_wait(&sm.accfull[a], use[a] & 1u, ctl, DETAIL_WAIT_ACCFULL);
      __syncwarp();
      tc_fence_after();
      const uint32_t taddr = tmem + a * 64 + ((wl * 32u) << 16);
      uint32_t ra[32], rb[32];
      tmem_ld_32x32b_x32(taddr, ra);
      tmem_ld_32x32b_x32(taddr + 32, rb);
      tmem_wait_ld_regs(ra);
      tmem_wait_ld_regs(rb);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.accempty[a]);
      ++use[a];
      float part[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int j = 0; j < 32; j += 4) {
        const float4 w0 = *reinterpret_cast<const float4*>(&sm.wq[j]);
        const float4 w1 = *reinterpret_cast<const float4*>(&sm.wq[32 + j]);
        part[0] = fmaf(w0.x, __saturatef(__uint_as_float(ra[j + 0]) * 0x1p-25f), part[0]);
        part[1] = fmaf(w0.y, __saturatef(__uint_as_float(ra[j + 1]) * 0x1p-25f), part[1]);
        part[2] = fmaf(w0.z, __saturatef(__uint_as_float(ra[j + 2]) * 0x1p-25f), part[2]);
        part[3] = fmaf(w0.w, __saturatef(__uint_as_float(ra[j + 3]) * 0x1p-25f), part[3]);
        part[0] = fmaf(w1.x, __saturatef(__uint_as_float(rb[j + 0]) * 0x1p-25f), part[0]);
        part[1] = fmaf(w1.y, __saturatef(__uint_as_float(rb[j + 1]) * 0x1p-25f), part[1]);
        part[2] = fmaf(w1.z, __saturatef(__uint_as_float(rb[j + 2]) * 0x1p-25f), part[2]);
        part[3] = fmaf(w1.w, __saturatef(__uint_as_float(rb[j + 3]) * 0x1p-25f), part[3]);
      }
      const float acc = (part[0] + part[1]) + (part[2] + part[3]);
      if (valid && got) {
        const float score = (acc * sq) * sk;
        out[s] = score;
        atomicAdd(&sm.hist[float_to_ordered(score + 0.0f) >> 21], 1u);
      }
      if (!__all_sync(0xFFFFFFFFu, got)) break;
    }
    named_bar(1, 128);
    uint32_t* gbins = p.bins + static_cast<size_t>(b) * kScoreBins;
    for (int i = rank; i < kScoreBins; i += 128) {
      const uint32_t c = sm.hist[i];
      if (c) atomicAdd(&gbins[i], c);
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

template <int D>
static dsa_status launch_decode_t(const DecodeLaunch& a) {
  using C = DCfg<D>;
  const size_t smem = sizeof(DSmem<D>) + 1024;
  auto kern = decode_indexer_kernel<D>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return DSA_ERR_CUDA;
  CUtensorMap tq, tk;
  if (!encode_tmap_2d_u8(&tq, a.q, D, static_cast<uint64_t>(a.B) * C::H, C::H)) return DSA_ERR_CUDA;
  if (!encode_tmap_2d_u8(&tk, a.k_cache, D, static_cast<uint64_t>(a.n_blocks) * C::PAGE, C::PAGE))
    return DSA_ERR_CUDA;
  const int max_len = a.max_blocks * a.block_size;
  DecodeParams p;
  p.q_scale = a.q_scale;
  p.w = a.w;
  p.k_scale_cache = a.k_scale_cache;
  p.block_table = a.block_table;
  p.seq_lens = a.seq_lens;
  p.max_blocks = a.max_blocks;
  p.n_blocks = a.n_blocks;
  p.max_len = max_len;
  uint8_t* base = static_cast<uint8_t*>(a.ws);
  const DecodeLayout lay = decode_layout(a.B, static_cast<size_t>(a.B) * max_len);
  p.hdr = reinterpret_cast<WsHeader*>(base);
  p.scores = reinterpret_cast<float*>(base + lay.scores);
  p.bins = reinterpret_cast<uint32_t*>(base + lay.bins);
  p.budget_ns = a.budget_ns;
  // Histograms and collection state, cleared together.
  if (cudaMemsetAsync(p.bins, 0, lay.cand - lay.bins, a.stream) != cudaSuccess) return DSA_ERR_CUDA;
  const int max_tiles = (max_len + C::BN - 1) / C::BN;
  dim3 grid((max_tiles + C::TPC - 1) / C::TPC, a.B);
  kern<<<grid, C::THREADS, smem, a.stream>>>(tq, tk, p);
  if (cudaGetLastError() != cudaSuccess) return DSA_ERR_CUDA;
  return launch_decode_topk(a.ws, lay, max_len, a.seq_lens, a.B, a.topk, a.out_idx, a.out_score,
                            a.budget_ns, a.stream);
}

size_t decode_workspace_bytes(int B, int max_len, int H, int d, int topk) {
  (void)H;
  (void)d;
  (void)topk;
  return decode_layout(B, static_cast<size_t>(B) * max_len).total;
}

dsa_status launch_decode(const DecodeLaunch& a) {
  if (a.H == 64 && a.d == 128 && a.block_size == 64) return launch_decode_t<128>(a);
  return DSA_ERR_UNSUPPORTED;
}

}  // namespace dsa

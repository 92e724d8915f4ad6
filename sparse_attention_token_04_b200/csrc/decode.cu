// Decode lightning indexer for sm_100a: one query (H = 64 heads) per request against its
// paged FP8 key cache.
//
// Persistent grid (as many CTAs as are resident at once). The requests' tiles (a tile being
// 128 logical keys = two 64-key pages), laid end to end in request order, are split into equal
// contiguous ranges, one per CTA, so every CTA streams the same number of tiles and none is
// launched or torn down in between. A range crosses a few requests; the part of it in one
// request is a segment. The work is HBM-bound (d + 4 bytes per key), so the CTA is small (three
// fit per SM) and keeps STAGES tiles in flight:
//   warp 0     TMA: per segment the request's 64 query rows (QBUF buffers; with one, the
//              next request's rows load once the current segment's MMAs are done), then per
//              tile the two pages named by the block table (entries are range-checked; a bad entry is
//              recorded as DSA_ERR_DEVICE and block 0 is read instead);
//   warp 1     one thread issues tcgen05.mma kind::f8f6f4, M = 128 keys, N = 64 heads,
//              K = d, into one of two 64-column TMEM accumulators;
//   warps 2-5  epilogue: thread = key; ReLU (on the FMA pipe, see prefill.cu), head weights,
//              scales; the score of every valid key is stored at scores[b][s] and counted in a
//              shared histogram of order-preserving top-11-bit bins, which is added to the
//              request's global histogram when the segment ends. The next request's head
//              weights and query scale are loaded a segment ahead.
// decode_collect_kernel and decode_rank_kernel (topk.cu) then select and order each request's
// top-k. Before the scoring kernel, decode_clear_kernel zeroes the histograms and the collection
// state; the scoring kernel is its programmatic dependent (its prologue and first tiles overlap
// the clear) and waits for it before its first histogram add and before it exits.
#include <algorithm>
#include <atomic>

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
  static constexpr int QBUF = 1;               // query-row buffers (1 keeps three CTAs per SM)
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
  uint8_t q[C::QBUF][C::QTILE];
  uint8_t k[C::STAGES][C::KTILE];
  float wq[C::H];
  uint32_t hist[kScoreBins];   // this segment's scores per order-preserving top-11-bit bin
  uint64_t kfull[C::STAGES];
  uint64_t kempty[C::STAGES];
  uint64_t qfull[C::QBUF], qempty[C::QBUF], accfull[2], accempty[2], drain;
  uint32_t tmem_base;
  int abort;
  int b0, tile0, ntiles;       // this CTA's range: first request, its first tile, tile count
};

struct DecodeParams {
  const float* q_scale;
  const float* w;
  const float* k_scale_cache;
  const int32_t* block_table;
  const int32_t* seq_lens;
  int32_t B, max_blocks, n_blocks, max_len;
  float* scores;
  uint32_t* bins;   // [B][kScoreBins] per-request score histogram
  WsHeader* hdr;
  uint64_t budget_ns;
};

// Request b's length, clamped to [1, max_len] (a bad length is recorded once, by CTA 0).
__device__ __forceinline__ int decode_len(const DecodeParams& p, int b) {
  const int n = __ldg(&p.seq_lens[b]);
  return n < 1 ? 1 : (n > p.max_len ? p.max_len : n);
}

template <int D>
__global__ void __launch_bounds__(192)
    decode_indexer_kernel(const __grid_constant__ CUtensorMap tmap_q,
                          const __grid_constant__ CUtensorMap tmap_k, const DecodeParams p) {
  using C = DCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  DSmem<D>& sm = *reinterpret_cast<DSmem<D>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t warp = threadIdx.x >> 5, lane = threadIdx.x & 31u;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&sm.kfull[s], 1);
      mbar_init(&sm.kempty[s], 1);
    }
    for (int a = 0; a < C::QBUF; ++a) {
      mbar_init(&sm.qfull[a], 1);
      mbar_init(&sm.qempty[a], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&sm.accfull[a], 1);
      mbar_init(&sm.accempty[a], 4);
    }
    mbar_init(&sm.drain, 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    // This CTA's range [lo, hi) of the T tiles of all requests, and the request holding lo.
    uint64_t T = 0;
    for (int base = 0; base < p.B; base += 32) {
      const int bb = base + static_cast<int>(lane);
      uint32_t nt = 0;
      if (bb < p.B) {
        const int raw = __ldg(&p.seq_lens[bb]);
        if ((raw < 1 || raw > p.max_len) && blockIdx.x == 0)
          record_error(p.hdr, DSA_ERR_DEVICE, DETAIL_BAD_SEQ_LEN);
        nt = static_cast<uint32_t>((decode_len(p, bb) + C::BN - 1) / C::BN);
      }
      T += __reduce_add_sync(0xFFFFFFFFu, nt);
    }
    const uint64_t lo = T * blockIdx.x / gridDim.x, hi = T * (blockIdx.x + 1) / gridDim.x;
    uint64_t carry = 0;
    bool found = false;
    for (int base = 0; base < p.B && lo < hi; base += 32) {
      const int bb = base + static_cast<int>(lane);
      const uint32_t nt = bb < p.B ? static_cast<uint32_t>((decode_len(p, bb) + C::BN - 1) / C::BN) : 0u;
      uint32_t incl = nt;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t o = __shfl_up_sync(0xFFFFFFFFu, incl, off);
        if (lane >= static_cast<uint32_t>(off)) incl += o;
      }
      const uint64_t start = carry + incl - nt;
      const uint32_t m = __ballot_sync(0xFFFFFFFFu, nt > 0 && start <= lo && lo < start + nt);
      if (m) {
        if (lane == static_cast<uint32_t>(__ffs(m) - 1)) {
          sm.b0 = bb;
          sm.tile0 = static_cast<int>(lo - start);
        }
        found = true;
        break;
      }
      carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
    }
    if (lane == 0) sm.ntiles = found ? static_cast<int>(hi - lo) : 0;
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

  auto phys_block = [&](const int32_t* table, int lb, bool record) -> int {
    int pb = __ldg(&table[lb]);
    if (pb < 0 || pb >= p.n_blocks) {
      if (record) record_error(p.hdr, DSA_ERR_DEVICE, DETAIL_BAD_BLOCK_TABLE);
      pb = 0;
    }
    return pb;
  };

  // Every role walks the same segments: request b, tiles [t, te), with `left` tiles of the
  // range after this segment.
  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tmap_q);
      prefetch_tmap(&tmap_k);
      // The key pages are read once; evicting them first keeps the scores this kernel writes
      // in L2 for the collection pass that reads them next.
      const uint64_t stream_policy = l2_policy_evict_first();
      uint32_t kiss[C::STAGES], qiss[C::QBUF];
      for (int s = 0; s < C::STAGES; ++s) kiss[s] = 0;
      for (int s = 0; s < C::QBUF; ++s) qiss[s] = 0;
      uint32_t gi = 0;
      bool stop = false;
      int b = sm.b0, t = sm.tile0, left = sm.ntiles;
      for (uint32_t j = 0; left > 0 && !stop; ++j, ++b, t = 0) {
        const int n = decode_len(p, b);
        const int te = min((n + C::BN - 1) / C::BN, t + left);
        left -= te - t;
        const uint32_t qs = j % C::QBUF;
        if (!mbar_wait(&sm.qempty[qs], ((j / C::QBUF) & 1u) ^ 1u, ctl, DETAIL_WAIT_QEMPTY)) break;
        mbar_arrive_expect_tx(&sm.qfull[qs], C::QTILE);
        tma_load_2d(sm.q[qs], &tmap_q, 0, b * C::H, &sm.qfull[qs]);
        ++qiss[qs];
        const int nblk = (n + C::PAGE - 1) / C::PAGE;
        const int32_t* table = p.block_table + static_cast<size_t>(b) * p.max_blocks;
        for (int tile = t; tile < te; ++tile, ++gi) {
          const uint32_t st = gi % C::STAGES, ph = (gi / C::STAGES) & 1u;
          if (!mbar_wait(&sm.kempty[st], ph ^ 1u, ctl, DETAIL_WAIT_KEMPTY)) {
            stop = true;
            break;
          }
          const int lb0 = 2 * tile, lb1 = 2 * tile + 1;
          const bool two = lb1 < nblk;
          mbar_arrive_expect_tx(&sm.kfull[st], two ? 2 * C::PAGE_BYTES : C::PAGE_BYTES);
          tma_load_2d_hint(sm.k[st], &tmap_k, 0, phys_block(table, lb0, true) * C::PAGE, &sm.kfull[st],
                           stream_policy);
          if (two)
            tma_load_2d_hint(sm.k[st] + C::PAGE_BYTES, &tmap_k, 0, phys_block(table, lb1, true) * C::PAGE,
                             &sm.kfull[st], stream_policy);
          ++kiss[st];
        }
      }
      // Let every copy this CTA issued land before it exits (bounded).
      for (int s = 0; s < C::STAGES; ++s)
        if (kiss[s]) mbar_wait_drain(&sm.kfull[s], (kiss[s] - 1) & 1u, p.budget_ns);
      for (int s = 0; s < C::QBUF; ++s)
        if (qiss[s]) mbar_wait_drain(&sm.qfull[s], (qiss[s] - 1) & 1u, p.budget_ns);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      uint32_t use[2] = {0, 0};
      uint32_t gi = 0;
      bool stop = false;
      int b = sm.b0, t = sm.tile0, left = sm.ntiles;
      for (uint32_t j = 0; left > 0 && !stop; ++j, ++b, t = 0) {
        const int n = decode_len(p, b);
        const int te = min((n + C::BN - 1) / C::BN, t + left);
        left -= te - t;
        const uint32_t qs = j % C::QBUF;
        if (!mbar_wait(&sm.qfull[qs], (j / C::QBUF) & 1u, ctl, DETAIL_WAIT_QFULL)) break;
        tc_fence_after();
        const uint32_t qa = smem_u32(sm.q[qs]);
        for (int tile = t; tile < te; ++tile, ++gi) {
          const uint32_t st = gi % C::STAGES, ph = (gi / C::STAGES) & 1u;
          const uint32_t a = gi & 1u;
          if (!mbar_wait(&sm.kfull[st], ph, ctl, DETAIL_WAIT_KFULL) ||
              !mbar_wait(&sm.accempty[a], (use[a] & 1u) ^ 1u, ctl, DETAIL_WAIT_ACCEMPTY)) {
            stop = true;
            break;
          }
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
        if (!stop) tc_commit(&sm.qempty[qs]);  // the query rows are free once these MMAs finish
      }
      tc_commit(&sm.drain);
      mbar_wait_drain(&sm.drain, 0, p.budget_ns);
    }
    __syncwarp();
  } else {
    // epilogue warps 2..5 -> TMEM lane quarters 2, 3, 0, 1
    const uint32_t wl = warp & 3u;
    const uint32_t rank = threadIdx.x - 64u;
    for (int i = rank; i < kScoreBins; i += 128) sm.hist[i] = 0u;
    int b = sm.b0, t = sm.tile0, left = sm.ntiles;
    float w_next = 0.0f, sq_next = 0.0f;
    if (left > 0) {
      if (rank < C::H) w_next = __ldg(&p.w[static_cast<size_t>(b) * C::H + rank]) * 0x1p25f;
      sq_next = __ldg(&p.q_scale[b]);
    }
    auto flush_hist = [&](int req) {
      grid_dependency_wait();  // the histograms are zero (decode_clear_kernel has completed)
      uint32_t* gbins = p.bins + static_cast<size_t>(req) * kScoreBins;
      for (int i = rank; i < kScoreBins; i += 128) {
        const uint32_t c = sm.hist[i];
        if (c) {
          atomicAdd(&gbins[i], c);
          sm.hist[i] = 0u;
        }
      }
    };
    uint32_t use[2] = {0, 0};
    uint32_t gi = 0, j = 0;
    bool stop = false;
    for (;; ++j, ++b, t = 0) {
      // Segment switch: every epilogue thread takes the same barriers, and all of them have
      // finished the previous segment (its histogram counts, its head weights).
      if (named_bar_or(1, 128, stop || left <= 0)) break;
      if (j > 0) flush_hist(b - 1);
      if (rank < C::H) sm.wq[rank] = w_next;
      const float sq = sq_next;
      const int n = decode_len(p, b);
      const int te = min((n + C::BN - 1) / C::BN, t + left);
      left -= te - t;
      named_bar(1, 128);
      if (left > 0) {
        if (rank < C::H) w_next = __ldg(&p.w[static_cast<size_t>(b + 1) * C::H + rank]) * 0x1p25f;
        sq_next = __ldg(&p.q_scale[b + 1]);
      }
      float* out = p.scores + static_cast<size_t>(b) * p.max_len;
      const int32_t* table = p.block_table + static_cast<size_t>(b) * p.max_blocks;
      // This thread's key scale, loaded one tile ahead.
      auto scale_of = [&](int s) {
        return s < n ? __ldcs(&p.k_scale_cache[static_cast<size_t>(phys_block(table, s / C::PAGE, false)) *
                                                   C::PAGE +
                                               (s % C::PAGE)])
                     : 0.0f;
      };
      float sk_next = scale_of(t * C::BN + static_cast<int>(wl * 32u + lane));
      for (int tile = t; tile < te; ++tile, ++gi) {
        const uint32_t a = gi & 1u;
        const int s = tile * C::BN + static_cast<int>(wl * 32u + lane);
        const bool valid = s < n;
        const float sk = sk_next;
        if (tile + 1 < te) sk_next = scale_of(s + C::BN);
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
        for (int jj = 0; jj < 32; jj += 4) {
          const float4 w0 = *reinterpret_cast<const float4*>(&sm.wq[jj]);
          const float4 w1 = *reinterpret_cast<const float4*>(&sm.wq[32 + jj]);
          part[0] = fmaf(w0.x, __saturatef(__uint_as_float(ra[jj + 0]) * 0x1p-25f), part[0]);
          part[1] = fmaf(w0.y, __saturatef(__uint_as_float(ra[jj + 1]) * 0x1p-25f), part[1]);
          part[2] = fmaf(w0.z, __saturatef(__uint_as_float(ra[jj + 2]) * 0x1p-25f), part[2]);
          part[3] = fmaf(w0.w, __saturatef(__uint_as_float(ra[jj + 3]) * 0x1p-25f), part[3]);
          part[0] = fmaf(w1.x, __saturatef(__uint_as_float(rb[jj + 0]) * 0x1p-25f), part[0]);
          part[1] = fmaf(w1.y, __saturatef(__uint_as_float(rb[jj + 1]) * 0x1p-25f), part[1]);
          part[2] = fmaf(w1.z, __saturatef(__uint_as_float(rb[jj + 2]) * 0x1p-25f), part[2]);
          part[3] = fmaf(w1.w, __saturatef(__uint_as_float(rb[jj + 3]) * 0x1p-25f), part[3]);
        }
        const float acc = (part[0] + part[1]) + (part[2] + part[3]);
        if (valid && got) {
          const float score = (acc * sq) * sk;
          out[s] = score;
          atomicAdd(&sm.hist[float_to_ordered(score + 0.0f) >> 21], 1u);
        }
        if (!__all_sync(0xFFFFFFFFu, got)) {
          stop = true;
          break;
        }
      }
    }
    if (j > 0) flush_hist(b - 1);
  }
  // Every CTA waits for the clear before it exits, so the kernels after this one, which wait
  // for this grid only, find the histograms and the collection state cleared.
  grid_dependency_wait();
  __syncthreads();
  grid_launch_dependents();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// Zeroes the per-request histograms and collection state (n words) and lets the scoring kernel
// launch at once.
__global__ void __launch_bounds__(256) decode_clear_kernel(uint32_t* __restrict__ words, uint32_t n) {
  grid_launch_dependents();
  for (uint32_t e = blockIdx.x * 256u + threadIdx.x; e < n; e += gridDim.x * 256u) words[e] = 0u;
}

// CTAs of the scoring kernel that fit on one SM at once (the persistent grid is this many per
// SM), from the SM's shared memory (less the per-CTA reservation), registers, threads and the
// 512 TMEM columns (128 per CTA). Computed once per device. Counting it here rather than with
// the occupancy query, which reported one CTA per SM where three were resident.
static int decode_ctas_per_sm(const void* kern, int threads, size_t smem) {
  static std::atomic<int> cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 0;
  if (dev < 64 && cached[dev].load() > 0) return cached[dev].load();
  int smem_sm = 0, reserved = 0, regs_sm = 0, threads_sm = 0;
  cudaFuncAttributes fa;
  if (cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&regs_sm, cudaDevAttrMaxRegistersPerMultiprocessor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&threads_sm, cudaDevAttrMaxThreadsPerMultiProcessor, dev) != cudaSuccess ||
      cudaFuncGetAttributes(&fa, kern) != cudaSuccess)
    return 0;
  const size_t per_cta_smem = smem + static_cast<size_t>(reserved) + fa.sharedSizeBytes;
  const int warp_regs = ((fa.numRegs * 32 + 255) / 256) * 256;  // allocated per warp, 256 at a time
  int n = static_cast<int>(static_cast<size_t>(smem_sm) / per_cta_smem);
  n = std::min(n, regs_sm / std::max(1, warp_regs * (threads / 32)));
  n = std::min(n, threads_sm / threads);
  n = std::min(n, 512 / 128);
  n = std::max(n, 1);
  if (dev < 64) cached[dev].store(n);
  return n;
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
  p.B = a.B;
  p.max_blocks = a.max_blocks;
  p.n_blocks = a.n_blocks;
  p.max_len = max_len;
  uint8_t* base = static_cast<uint8_t*>(a.ws);
  const DecodeLayout lay = decode_layout(a.B, static_cast<size_t>(a.B) * max_len);
  p.hdr = reinterpret_cast<WsHeader*>(base);
  p.scores = reinterpret_cast<float*>(base + lay.scores);
  p.bins = reinterpret_cast<uint32_t*>(base + lay.bins);
  p.budget_ns = a.budget_ns;
  // Histograms and collection state, cleared together by a small kernel whose programmatic
  // dependent is the scoring kernel.
  const uint32_t n_clear = static_cast<uint32_t>((lay.cand - lay.bins) / sizeof(uint32_t));
  const uint32_t clear_grid = std::min<uint32_t>((n_clear + 1023u) / 1024u, 128u);
  decode_clear_kernel<<<clear_grid, 256, 0, a.stream>>>(p.bins, n_clear);
  if (cudaGetLastError() != cudaSuccess) return DSA_ERR_CUDA;
  const int per_sm = decode_ctas_per_sm(reinterpret_cast<const void*>(kern), C::THREADS, smem);
  if (per_sm < 1) return DSA_ERR_CUDA;
  const int grid = per_sm * (a.num_sms > 0 ? a.num_sms : 1);
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(C::THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = a.stream;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, tq, tk, p) != cudaSuccess) return DSA_ERR_CUDA;
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

// Sparse-attention consumer of the decode index buffer for sm_100a: the core MLA attention of
// one decode query per request over only its k selected latents ("Index Share逻辑详解" §2: the
// indexer scores the whole length, the top-k is selected, and the core MLA attention runs on
// those k latents).
//
// Shapes: 128 query heads, a 576-wide bf16 latent (the keys), whose first 512 entries are the
// values. For request b and head h:
//     out[b, h] = sum_s softmax_s(scale * q[b, h] . K[s]) V[s]  over the selected positions s.
//
// attention_split_kernel: CTA (c, b) takes the 256 selected positions c*256 .. c*256+255 of
// request b. All operands are bf16 tiles in shared memory with the 128-byte swizzle, written by
// cp.async (zero-filled for unselected keys), and every product runs on the tensor cores
// (tcgen05.mma kind::f16, FP32 accumulators in TMEM):
//   1. S[128 heads][256 keys] = Q . K^T over the 576 dims, nine 64-dim chunks in three stages,
//      loaded two chunks ahead (each chunk: four M=128, N=256, K=16 MMAs into TMEM columns
//      0..255);
//   2. the loads of the first four value chunks start, then all eight warps read S (warp w:
//      heads 32(w%4).., keys 128(w/4)..), mask unselected keys and form the split's softmax
//      numerators P = exp(scale (S - m)) in bf16 (shared memory, K-major), with the row max m
//      and the two partial sums of l exchanged through shared memory;
//   3. O[128][512] = P . V over eight 32-key chunks: each chunk holds its keys' 512 value dims
//      as they sit in the latent row (dims contiguous, the MN-major operand layout, no
//      transposes), four slots of 32 KB loaded up to three chunks ahead; dims 0..255 accumulate
//      in TMEM columns 256..511 and dims 256..511 in columns 0..255, which S no longer needs;
//   4. warps 0..3 write O's first half, warps 4..7 its second, unnormalised, with m and l, to
//      the workspace.
// attention_combine_kernel then merges the splits of a request (log-sum-exp weights) into out.
// Waits on the tensor core are bounded; a timeout is recorded as DSA_ERR_TIMEOUT.
#include <algorithm>
#include <cmath>

#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"

namespace dsa {

constexpr int kAttHeads = 128;
constexpr int kAttDqk = 576;
constexpr int kAttDv = 512;
constexpr int kAttHalf = 256;             // value dims per accumulator (N of one MMA)
constexpr int kAttSplit = 256;            // selected keys per CTA
constexpr int kAttChunk = 64;             // dims per QK chunk (128-byte rows)
constexpr int kAttThreads = 256;
constexpr int kAttQkChunks = kAttDqk / kAttChunk;   // 9
constexpr int kAttQkStages = 3;
constexpr int kAttPvKeys = 32;                       // keys per value chunk
constexpr int kAttPvChunks = kAttSplit / kAttPvKeys;  // 8
constexpr int kAttPvSlots = 4;
constexpr int kAttPvSlotBytes = kAttPvKeys * kAttDv * 2;  // 32 KB
constexpr int kAttPvBlockBytes = kAttPvKeys * 128;         // one 64-dim column block of a chunk

struct AttSmem {
  // QK stages: Q chunk [128][64] + K chunk [256][64] bf16 each (48 KB); once S is complete the
  // first 128 KB hold the four value slots, each [8 column blocks of 64 dims][32 keys][64 dims].
  uint8_t stage[kAttQkStages][48 * 1024];
  uint8_t p[kAttSplit / 64][kAttHeads * 128];  // P [128 heads][256 keys] as four K-major 64-key chunks
  int32_t rows[kAttSplit];                     // latent row of each selected key, -1: masked
  float pm[2][kAttHeads], pl[2][kAttHeads];    // per key half: row max, sum of the rounded weights
  uint64_t qk_done[kAttQkStages], pv_done[kAttPvSlots];
  uint32_t tmem;
  int abort;
};
static_assert(kAttPvSlots * kAttPvSlotBytes <= kAttQkStages * 48 * 1024, "value slots exceed the stages");

__host__ __device__ constexpr uint32_t make_idesc_bf16(uint32_t M, uint32_t N) {
  return (1u << 4)                 // D format F32
         | (1u << 7) | (1u << 10)  // A, B format BF16
         | ((N >> 3) << 17)        // N / 8
         | ((M >> 4) << 24);       // M / 16
}
constexpr uint32_t kIdescBMnMajor = 1u << 16;  // B operand MN-major (N contiguous)

// Shared-memory descriptor of an MN-major operand with the 128-byte swizzle: rows of 64
// contiguous MN elements (128 bytes), eight K rows per 1024-byte atom; sbo = bytes between
// groups of eight K rows, lbo = bytes between 64-element MN column blocks.
__device__ __forceinline__ uint64_t make_smem_desc_mn(uint32_t smem_addr, uint32_t lbo, uint32_t sbo) {
  uint64_t desc = 0;
  desc |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);
  desc |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  desc |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  desc |= 1ull << 46;  // descriptor version
  desc |= 2ull << 61;  // 128-byte swizzle
  return desc;
}

__device__ __forceinline__ void tc_mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 16-byte cp.async; src_bytes = 0 fills the destination with zeros.
__device__ __forceinline__ void cp_async_16(void* smem_dst, const void* gsrc, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem_dst)), "l"(gsrc),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Byte offset of 16-byte unit u of row r in a K-major tile of 128-byte rows with the 128-byte
// swizzle (eight rows per 1024-byte atom, unit index XOR row index).
__device__ __forceinline__ uint32_t sw128(uint32_t r, uint32_t u) {
  return (r >> 3) * 1024u + (r & 7u) * 128u + ((u ^ (r & 7u)) << 4);
}

struct AttParams {
  const uint16_t* q;          // [B][128][576] bf16
  const uint16_t* latent;     // [n_blocks * block_size][576] bf16
  const int32_t* block_table; // [B][max_blocks]
  const int32_t* seq_lens;    // [B]
  const int32_t* idx;         // [B][topk]
  int32_t n_blocks, block_size, max_blocks, B, topk;
  float scale_log2;           // scale * log2(e)
  float* o_part;              // [B][n_split][512 dims][128 heads]
  float* ml;                  // [B][n_split][2][128]
  WsHeader* hdr;
  uint64_t budget_ns;
};

__global__ void __launch_bounds__(kAttThreads, 1) attention_split_kernel(const __grid_constant__ AttParams p) {
  extern __shared__ uint8_t smem_raw[];
  AttSmem& sm = *reinterpret_cast<AttSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  const uint32_t tid = threadIdx.x, warp = tid >> 5, lane = tid & 31u;
  const int c = blockIdx.x, b = blockIdx.z;
  const int n_split = gridDim.x;
  if (tid == 0) {
    for (int i = 0; i < kAttQkStages; ++i) mbar_init(&sm.qk_done[i], 1);
    for (int i = 0; i < kAttPvSlots; ++i) mbar_init(&sm.pv_done[i], 1);
    fence_mbar_init();
    sm.abort = 0;
  }
  if (warp == 0) {
    tmem_alloc(&sm.tmem, 512);
    tmem_relinquish();
  }
  // The split's keys: logical position -> latent row (checked), -1 for none.
  {
    int n = p.seq_lens[b];
    const bool bad_len = n < 1 || n > p.max_blocks * p.block_size;
    n = bad_len ? 0 : n;
    const int s = p.idx[static_cast<size_t>(b) * p.topk + c * kAttSplit + tid];
    int row = -1;
    bool bad = bad_len && tid == 0;
    if (s >= 0 && s < n) {
      const int blk = p.block_table[static_cast<size_t>(b) * p.max_blocks + s / p.block_size];
      if (blk >= 0 && blk < p.n_blocks) row = blk * p.block_size + s % p.block_size;
      else bad = true;
    } else if (s != -1) {
      bad = true;
    }
    if (bad) record_error(p.hdr, DSA_ERR_DEVICE, DETAIL_BAD_INDEX);
    sm.rows[tid] = row;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem;
  const uint32_t tS = tmem, tO = tmem + kAttSplit;
  const WaitCtl ctl{p.hdr, &sm.abort, p.budget_ns};
  const uint16_t* qb = p.q + static_cast<size_t>(b) * kAttHeads * kAttDqk;
  bool ok = true;
  uint32_t qk_issued[kAttQkStages] = {0, 0, 0}, pv_issued[kAttPvSlots] = {0, 0, 0, 0};

  // 1. S = Q K^T over nine 64-dim chunks, loads two chunks ahead of the MMAs (three stages).
  auto load_qk = [&](int ch) {
    const int st = ch % kAttQkStages;
    uint8_t* qs = sm.stage[st];
    uint8_t* ks = sm.stage[st] + kAttHeads * 128;
#pragma unroll
    for (int i = 0; i < 4; ++i) {  // Q chunk: 128 rows x 8 units
      const uint32_t u = tid + i * kAttThreads, r = u >> 3, j = u & 7u;
      cp_async_16(qs + sw128(r, j), qb + static_cast<size_t>(r) * kAttDqk + ch * kAttChunk + j * 8, 16);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {  // K chunk: 256 rows x 8 units
      const uint32_t u = tid + i * kAttThreads, r = u >> 3, j = u & 7u;
      const int row = sm.rows[r];
      const uint16_t* src = p.latent + static_cast<size_t>(row < 0 ? 0 : row) * kAttDqk + ch * kAttChunk + j * 8;
      cp_async_16(ks + sw128(r, j), src, row < 0 ? 0u : 16u);
    }
    cp_async_commit();
  };
  load_qk(0);
  load_qk(1);
  for (int ch = 0; ch < kAttQkChunks && ok; ++ch) {
    const int st = ch % kAttQkStages;
    if (ch + 2 < kAttQkChunks) {
      // stage (ch + 2) % 3 was last read by the MMAs of chunk ch - 1
      const int sn = (ch + 2) % kAttQkStages;
      if (qk_issued[sn] > 0) ok = mbar_wait(&sm.qk_done[sn], (qk_issued[sn] - 1) & 1u, ctl, DETAIL_WAIT_ACCFULL);
      if (__syncthreads_or(!ok)) { ok = false; break; }
      load_qk(ch + 2);
      cp_async_wait<2>();  // this thread's copies of chunk ch have landed
    } else if (ch + 1 < kAttQkChunks) {
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      const uint64_t da = make_smem_desc(smem_u32(sm.stage[st]), 128);
      const uint64_t db = make_smem_desc(smem_u32(sm.stage[st] + kAttHeads * 128), 128);
#pragma unroll
      for (int kk = 0; kk < kAttChunk / 16; ++kk)
        tc_mma_bf16(tS, da + 2ull * kk, db + 2ull * kk, make_idesc_bf16(kAttHeads, kAttSplit),
                    (ch > 0 || kk > 0) ? 1u : 0u);
      tc_commit(&sm.qk_done[st]);
    }
    ++qk_issued[st];
  }
  cp_async_wait<0>();  // nothing of this CTA's is still landing (also on the abort path)
  // S complete: the last chunk's commit covers every earlier MMA, so the stages are free.
  const int last_qk = (kAttQkChunks - 1) % kAttQkStages;
  if (ok) ok = mbar_wait(&sm.qk_done[last_qk], (qk_issued[last_qk] - 1) & 1u, ctl, DETAIL_WAIT_ACCFULL);
  ok = !__syncthreads_or(!ok);

  // Value chunk i: keys i*32 .. i*32+31, all 512 value dims, into slot i % 4 as eight 64-dim
  // column blocks of [32 keys][128 bytes]; a warp copies 512 contiguous bytes of one key.
  auto load_v = [&](int i) {
    uint8_t* slot = sm.stage[0] + (i % kAttPvSlots) * kAttPvSlotBytes;
#pragma unroll
    for (int it = 0; it < kAttPvSlotBytes / 16 / kAttThreads; ++it) {  // 8
      const uint32_t u = tid + it * kAttThreads, r = u >> 6, j = u & 63u;
      const int row = sm.rows[i * kAttPvKeys + r];
      const uint16_t* src = p.latent + static_cast<size_t>(row < 0 ? 0 : row) * kAttDqk + j * 8;
      cp_async_16(slot + (j >> 3) * kAttPvBlockBytes + sw128(r, j & 7u), src, row < 0 ? 0u : 16u);
    }
    cp_async_commit();
  };
  if (ok) {
#pragma unroll
    for (int i = 0; i < kAttPvSlots; ++i) load_v(i);
  }

  // 2. Softmax numerators of the split: warp w takes heads 32(w%4).. over keys 128(w/4)..
  const uint32_t h = (warp & 3u) * 32u + lane, kh = warp >> 2;
  const uint32_t lane_base = ((warp & 3u) * 32u) << 16;
  if (ok) {
    tc_fence_after();
    float mx = -INFINITY;
#pragma unroll 1
    for (int cc = 0; cc < 4; ++cc) {
      const int key0 = kh * 128 + cc * 32;
      uint32_t r[32];
      tmem_ld_32x32b_x32(tS + lane_base + key0, r);
      tmem_wait_ld_regs(r);
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (sm.rows[key0 + j] >= 0) mx = fmaxf(mx, __uint_as_float(r[j]));
    }
    sm.pm[kh][h] = mx;
    __syncthreads();
    mx = fmaxf(sm.pm[0][h], sm.pm[1][h]);
    float sum = 0.0f;
#pragma unroll 1
    for (int cc = 0; cc < 4; ++cc) {
      const int key0 = kh * 128 + cc * 32;
      uint32_t r[32];
      tmem_ld_32x32b_x32(tS + lane_base + key0, r);
      tmem_wait_ld_regs(r);
      uint32_t packed[16];
#pragma unroll
      for (int j = 0; j < 32; j += 2) {
        const bool v0 = sm.rows[key0 + j] >= 0, v1 = sm.rows[key0 + j + 1] >= 0;
        const float p0 = v0 ? exp2f((__uint_as_float(r[j]) - mx) * p.scale_log2) : 0.0f;
        const float p1 = v1 ? exp2f((__uint_as_float(r[j + 1]) - mx) * p.scale_log2) : 0.0f;
        const __nv_bfloat162 pp = __floats2bfloat162_rn(p0, p1);
        sum += __low2float(pp) + __high2float(pp);  // the weights the value product uses
        packed[j >> 1] = *reinterpret_cast<const uint32_t*>(&pp);
      }
      // keys key0 .. key0+31: P chunk key0/64, units (key0/32 & 1)*4 .. +3 of row h
      uint8_t* pc = sm.p[key0 >> 6];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint4 w4 = make_uint4(packed[4 * u], packed[4 * u + 1], packed[4 * u + 2], packed[4 * u + 3]);
        *reinterpret_cast<uint4*>(pc + sw128(h, ((key0 >> 5) & 1) * 4 + u)) = w4;
      }
    }
    sm.pl[kh][h] = sum;
    tc_fence_before();
  }
  fence_proxy_async_smem();

  // 3. O = P V over eight 32-key chunks; dims 0..255 into columns 256..511, dims 256..511 into
  // columns 0..255. After issuing chunk i (1 <= i <= 4), slot (i-1) % 4 is refilled with chunk
  // i+3 once the MMAs of chunk i-1 have read it.
  const uint32_t idesc_pv = make_idesc_bf16(kAttHeads, kAttHalf) | kIdescBMnMajor;
#pragma unroll 1
  for (int i = 0; i < kAttPvChunks && ok; ++i) {
    // this thread's copies of chunk i have landed; the newer groups may still be in flight
    if (i == 0) cp_async_wait<3>();
    else if (i <= 5) cp_async_wait<2>();
    else if (i == 6) cp_async_wait<1>();
    else cp_async_wait<0>();
    fence_proxy_async_smem();
    if (__syncthreads_or(!ok)) { ok = false; break; }
    const int slot = i % kAttPvSlots;
    if (tid == 0) {
      tc_fence_after();
      const uint32_t vbase = smem_u32(sm.stage[0] + slot * kAttPvSlotBytes);
      const uint64_t da = make_smem_desc(smem_u32(sm.p[i >> 1]), 128);
#pragma unroll
      for (int half = 0; half < kAttDv / kAttHalf; ++half) {
#pragma unroll
        for (int kk = 0; kk < kAttPvKeys / 16; ++kk) {
          const uint64_t db = make_smem_desc_mn(vbase + half * 4 * kAttPvBlockBytes + kk * 2048,
                                                kAttPvBlockBytes, 1024);
          tc_mma_bf16(half == 0 ? tO : tS, da + 2ull * ((i & 1) * 2 + kk), db, idesc_pv,
                      (i > 0 || kk > 0) ? 1u : 0u);
        }
      }
      tc_commit(&sm.pv_done[slot]);
    }
    ++pv_issued[slot];
    if (i >= 1 && i + 3 < kAttPvChunks) {
      const int sp = (i - 1) % kAttPvSlots;
      ok = mbar_wait(&sm.pv_done[sp], (pv_issued[sp] - 1) & 1u, ctl, DETAIL_WAIT_ACCFULL);
      if (__syncthreads_or(!ok)) { ok = false; break; }
      load_v(i + 3);
    }
  }
  cp_async_wait<0>();
  const int last_pv = (kAttPvChunks - 1) % kAttPvSlots;
  if (ok) ok = mbar_wait(&sm.pv_done[last_pv], (pv_issued[last_pv] - 1) & 1u, ctl, DETAIL_WAIT_ACCFULL);
  ok = !__syncthreads_or(!ok);

  // 4. The unnormalised O of the split with m and l: warps 0..3 dims 0..255 (columns
  // 256..511), warps 4..7 dims 256..511 (columns 0..255). The partials are stored dim-major
  // ([dim][head]), so each store of a warp writes 128 contiguous bytes.
  if (ok) {
    tc_fence_after();
    float* dst = p.o_part + ((static_cast<size_t>(b) * n_split + c) * kAttDv + kh * kAttHalf) * kAttHeads + h;
    const uint32_t tcol = kh == 0 ? tO : tS;
#pragma unroll 1
    for (int cc = 0; cc < kAttHalf / 32; ++cc) {
      uint32_t r[32];
      tmem_ld_32x32b_x32(tcol + lane_base + cc * 32, r);
      tmem_wait_ld_regs(r);
#pragma unroll
      for (int j = 0; j < 32; ++j) dst[(cc * 32 + j) * kAttHeads] = __uint_as_float(r[j]);
    }
    if (kh == 0) {
      float* ml = p.ml + (static_cast<size_t>(b) * n_split + c) * 2 * kAttHeads;
      ml[h] = fmaxf(sm.pm[0][h], sm.pm[1][h]);
      ml[kAttHeads + h] = sm.pl[0][h] + sm.pl[1][h];
    }
    tc_fence_before();
  }
  if (!ok && tid == 0) {
    // Let the MMAs this CTA issued land before its TMEM is freed (bounded).
    for (int i = 0; i < kAttQkStages; ++i)
      if (qk_issued[i]) mbar_wait_drain(&sm.qk_done[i], (qk_issued[i] - 1) & 1u, p.budget_ns);
    for (int i = 0; i < kAttPvSlots; ++i)
      if (pv_issued[i]) mbar_wait_drain(&sm.pv_done[i], (pv_issued[i] - 1) & 1u, p.budget_ns);
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// out[b][h][d] = sum_c e^(m_c - M) O_c[h][d] / sum_c e^(m_c - M) l_c over the request's splits
// (M the largest m_c); a head whose splits selected nothing gets zeros. Block (x, b) takes dims
// 16x .. 16x+15 of all 128 heads: the partials are read along heads, 16 bytes a thread with
// every split's loads in flight at once, and out is written in 64-byte runs.
constexpr int kCombineDims = 16;
constexpr int kMaxSplits = DSA_MAX_TOPK / kAttSplit;
template <int NS>
__global__ void __launch_bounds__(256) attention_combine_kernel(const float* __restrict__ o_part,
                                                                const float* __restrict__ ml,
                                                                float scale_log2, float* __restrict__ out) {
  constexpr int n_split = NS;
  __shared__ __align__(16) float wt[NS][kAttHeads];
  __shared__ float tile[kCombineDims][kAttHeads + 1];
  const int d0 = blockIdx.x * kCombineDims, b = blockIdx.y;
  const int tid = threadIdx.x;
  static_assert(NS >= 1 && NS <= kMaxSplits, "splits per request");
  const float* mlb = ml + static_cast<size_t>(b) * n_split * 2 * kAttHeads;
  if (tid < kAttHeads) {
    const int h = tid;
    float mc[NS], lc[NS];
#pragma unroll
    for (int c = 0; c < NS; ++c) {
      mc[c] = mlb[c * 2 * kAttHeads + h];
      lc[c] = mlb[c * 2 * kAttHeads + kAttHeads + h];
    }
    float M = -INFINITY;
#pragma unroll
    for (int c = 0; c < NS; ++c) M = fmaxf(M, mc[c]);
    float wsum = 0.0f;
#pragma unroll
    for (int c = 0; c < NS; ++c) {
      mc[c] = (mc[c] == -INFINITY) ? 0.0f : exp2f((mc[c] - M) * scale_log2);
      wsum += mc[c] * lc[c];
    }
    const float inv = wsum > 0.0f ? 1.0f / wsum : 0.0f;
#pragma unroll
    for (int c = 0; c < NS; ++c) wt[c][h] = mc[c] * inv;
  }
  __syncthreads();
  {
    // thread: heads 4(t%32) .. +3, dims d0 + 2(t/32), +1; a warp reads 512 contiguous bytes
    const int hq = tid & 31, dd = tid >> 5;
    const float* src = o_part + (static_cast<size_t>(b) * n_split * kAttDv + d0 + 2 * dd) * kAttHeads + 4 * hq;
    float4 v[NS][2];
#pragma unroll
    for (int c = 0; c < NS; ++c)
#pragma unroll
      for (int j = 0; j < 2; ++j)
        v[c][j] = __ldcs(reinterpret_cast<const float4*>(src + (static_cast<size_t>(c) * kAttDv + j) * kAttHeads));
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
      for (int c = 0; c < NS; ++c) {
        const float4 w = *reinterpret_cast<const float4*>(&wt[c][4 * hq]);
        acc.x += w.x * v[c][j].x;
        acc.y += w.y * v[c][j].y;
        acc.z += w.z * v[c][j].z;
        acc.w += w.w * v[c][j].w;
      }
      float* trow = tile[2 * dd + j] + 4 * hq;
      trow[0] = acc.x;
      trow[1] = acc.y;
      trow[2] = acc.z;
      trow[3] = acc.w;
    }
  }
  __syncthreads();
  const int lane = tid & 31, warp = tid >> 5;
  for (int h = warp * 2 + (lane >> 4); h < kAttHeads; h += 16)
    out[(static_cast<size_t>(b) * kAttHeads + h) * kAttDv + d0 + (lane & 15)] = tile[lane & 15][h];
}

size_t attention_workspace_bytes(int B, int topk) {
  const size_t n_split = static_cast<size_t>(topk) / kAttSplit;
  const size_t o = static_cast<size_t>(B) * n_split * kAttHeads * kAttDv * sizeof(float);
  const size_t ml = static_cast<size_t>(B) * n_split * 2 * kAttHeads * sizeof(float);
  return DSA_WS_HEADER_BYTES + o + ml;
}

dsa_status launch_attention(const AttentionLaunch& a) {
  const int n_split = a.topk / kAttSplit;
  if (n_split < 1 || n_split > kMaxSplits || a.topk % kAttSplit != 0) return DSA_ERR_UNSUPPORTED;
  uint8_t* base = static_cast<uint8_t*>(a.ws);
  AttParams p;
  p.q = a.q;
  p.latent = a.latent;
  p.block_table = a.block_table;
  p.seq_lens = a.seq_lens;
  p.idx = a.idx;
  p.n_blocks = a.n_blocks;
  p.block_size = a.block_size;
  p.max_blocks = a.max_blocks;
  p.B = a.B;
  p.topk = a.topk;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.hdr = reinterpret_cast<WsHeader*>(base);
  p.o_part = reinterpret_cast<float*>(base + DSA_WS_HEADER_BYTES);
  p.ml = p.o_part + static_cast<size_t>(a.B) * n_split * kAttHeads * kAttDv;
  p.budget_ns = a.budget_ns;
  const size_t smem = sizeof(AttSmem) + 1024;
  if (cudaFuncSetAttribute(attention_split_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return DSA_ERR_CUDA;
  attention_split_kernel<<<dim3(n_split, 1, a.B), kAttThreads, smem, a.stream>>>(p);
  if (cudaGetLastError() != cudaSuccess) return DSA_ERR_CUDA;
  const dim3 cgrid(kAttDv / kCombineDims, a.B);
  switch (n_split) {
#define DSA_COMBINE_CASE(NS)                                                                   \
  case NS:                                                                                     \
    attention_combine_kernel<NS><<<cgrid, 256, 0, a.stream>>>(p.o_part, p.ml, p.scale_log2, a.out); \
    break;
    DSA_COMBINE_CASE(1) DSA_COMBINE_CASE(2) DSA_COMBINE_CASE(3) DSA_COMBINE_CASE(4)
    DSA_COMBINE_CASE(5) DSA_COMBINE_CASE(6) DSA_COMBINE_CASE(7) DSA_COMBINE_CASE(8)
#undef DSA_COMBINE_CASE
    default: return DSA_ERR_UNSUPPORTED;
  }
  return cuda_status(cudaGetLastError());
}

}  // namespace dsa

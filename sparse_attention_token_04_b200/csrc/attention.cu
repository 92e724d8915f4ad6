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
// request b. All operands are K-major bf16 tiles
// in shared memory with the 128-byte swizzle, written by the CTA's threads (cp.async for the
// query and key rows, register transposes for the values), and every product runs on the
// tensor cores (tcgen05.mma kind::f16, FP32 accumulators in TMEM):
//   1. S[128 heads][256 keys] = Q . K^T over the 576 dims, nine 64-dim chunks in three stages,
//      loaded two chunks ahead (each chunk: four M=128, N=256, K=16 MMAs into TMEM columns
//      0..255);
//   2. four warps (thread = head) read S, mask unselected keys, and form the split's softmax
//      numerators P = exp(scale (S - m)) in bf16 (shared memory, K-major) with the row max m
//      and sum l in fp32;
//   3. for each value half (dims 0..255, then 256..511): O[128][256] = P . V over the 256 keys,
//      four 64-key chunks whose V^T tiles are built by transposing 8x8 blocks in registers
//      (MMAs into TMEM columns 256..511, which S no longer needs), and the half of O goes to the
//      workspace; m and l go with the first half.
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
constexpr int kAttHalf = 256;             // value dims per CTA
constexpr int kAttSplit = 256;            // selected keys per CTA
constexpr int kAttChunk = 64;             // dims per QK chunk, keys per PV chunk (128-byte rows)
constexpr int kAttThreads = 256;
constexpr int kAttQkChunks = kAttDqk / kAttChunk;   // 9
constexpr int kAttPvChunks = kAttSplit / kAttChunk;  // 4

constexpr int kAttQkStages = 3;

struct AttSmem {
  // QK stages: Q chunk [128][64] + K chunk [256][64] bf16 each (48 KB); the two V^T stages
  // [256 dims][64 keys] (32 KB each) reuse them once S is complete.
  uint8_t stage[kAttQkStages][48 * 1024];
  uint8_t p[kAttPvChunks][kAttHeads * 128];  // P [128 heads][256 keys] as four K-major 64-key chunks
  int32_t rows[kAttSplit];                   // latent row of each selected key, -1: masked
  float m[kAttHeads], l[kAttHeads];
  uint64_t qk_done[kAttQkStages], pv_done[2];
  uint32_t tmem;
  int abort;
};

__host__ __device__ constexpr uint32_t make_idesc_bf16(uint32_t M, uint32_t N) {
  return (1u << 4)                 // D format F32
         | (1u << 7) | (1u << 10)  // A, B format BF16
         | ((N >> 3) << 17)        // N / 8
         | ((M >> 4) << 24);       // M / 16
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
  float* o_part;              // [B][n_split][128][512]
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
    for (int i = 0; i < 2; ++i) mbar_init(&sm.pv_done[i], 1);
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
  uint32_t qk_issued[kAttQkStages] = {0, 0, 0}, pv_issued[2] = {0, 0};

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
  // S complete: the last chunk's commit covers every earlier MMA.
  const int last_qk = (kAttQkChunks - 1) % kAttQkStages;
  if (ok) ok = mbar_wait(&sm.qk_done[last_qk], (qk_issued[last_qk] - 1) & 1u, ctl, DETAIL_WAIT_ACCFULL);
  ok = !__syncthreads_or(!ok);

  // 2. Softmax numerators of the split (warps 0..3, thread = head).
  if (ok && warp < 4) {
    tc_fence_after();
    const uint32_t h = warp * 32u + lane;
    const uint32_t lane_base = (warp * 32u) << 16;
    float mx = -INFINITY;
    for (int cc = 0; cc < kAttSplit / 32; ++cc) {
      uint32_t r[32];
      tmem_ld_32x32b_x32(tS + lane_base + cc * 32, r);
      tmem_wait_ld_regs(r);
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (sm.rows[cc * 32 + j] >= 0) mx = fmaxf(mx, __uint_as_float(r[j]));
    }
    float sum = 0.0f;
    for (int cc = 0; cc < kAttSplit / 32; ++cc) {
      uint32_t r[32];
      tmem_ld_32x32b_x32(tS + lane_base + cc * 32, r);
      tmem_wait_ld_regs(r);
      uint32_t packed[16];
#pragma unroll
      for (int j = 0; j < 32; j += 2) {
        const bool v0 = sm.rows[cc * 32 + j] >= 0, v1 = sm.rows[cc * 32 + j + 1] >= 0;
        const float p0 = v0 ? exp2f((__uint_as_float(r[j]) - mx) * p.scale_log2) : 0.0f;
        const float p1 = v1 ? exp2f((__uint_as_float(r[j + 1]) - mx) * p.scale_log2) : 0.0f;
        const __nv_bfloat162 pp = __floats2bfloat162_rn(p0, p1);
        sum += __low2float(pp) + __high2float(pp);  // the weights the value product uses
        packed[j >> 1] = *reinterpret_cast<const uint32_t*>(&pp);
      }
      // keys cc*32 .. cc*32+31: chunk cc/2, units (cc&1)*4 .. +3 of row h
      uint8_t* pc = sm.p[cc >> 1];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint4 w4 = make_uint4(packed[4 * u], packed[4 * u + 1], packed[4 * u + 2], packed[4 * u + 3]);
        *reinterpret_cast<uint4*>(pc + sw128(h, (cc & 1) * 4 + u)) = w4;
      }
    }
    sm.m[h] = mx;
    sm.l[h] = sum;
    tc_fence_before();
  }
  fence_proxy_async_smem();
  __syncthreads();

  // 3. and 4., once per value half v: O = P V over four 64-key chunks into TMEM columns
  // 256..511 (V^T chunks built by 8x8 register transposes, the next chunk's rows loading while
  // the current one is transposed), then the unnormalised O of the half to the workspace.
  const uint32_t ko = tid & 7u, dO = tid >> 3;  // key octet, dim octet (32 of them: 256 dims)
  auto load_v = [&](int v, int kc, uint4 (&x)[8]) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int row = sm.rows[kc * kAttChunk + ko * 8 + i];
      x[i] = row < 0 ? make_uint4(0u, 0u, 0u, 0u)
                     : __ldg(reinterpret_cast<const uint4*>(p.latent + static_cast<size_t>(row) * kAttDqk +
                                                            v * kAttHalf + dO * 8));
    }
  };
  uint4 xa[8], xb[8];
  for (int v = 0; v < kAttDv / kAttHalf && ok; ++v) {
    load_v(v, 0, xa);
    for (int kc = 0; kc < kAttPvChunks && ok; ++kc) {
      const int st = kc & 1;
      if (pv_issued[st] > 0) ok = mbar_wait(&sm.pv_done[st], (pv_issued[st] - 1) & 1u, ctl, DETAIL_WAIT_ACCFULL);
      if (__syncthreads_or(!ok)) { ok = false; break; }
      if (kc + 1 < kAttPvChunks) load_v(v, kc + 1, xb);
      uint8_t* vt = sm.stage[st];  // [256 dims][64 keys]
      // xa[i] holds dims dO*8 .. +7 of key i; row e of the block gathers dim e of keys 0..7.
      const uint32_t* xw = reinterpret_cast<const uint32_t*>(xa);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        uint32_t w[4];
#pragma unroll
        for (int k2 = 0; k2 < 4; ++k2) {
          const uint32_t a = xw[(2 * k2) * 4 + (e >> 1)], bb = xw[(2 * k2 + 1) * 4 + (e >> 1)];
          w[k2] = __byte_perm(a, bb, (e & 1) ? 0x7632u : 0x5410u);
        }
        *reinterpret_cast<uint4*>(vt + sw128(dO * 8 + e, ko)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      fence_proxy_async_smem();
      __syncthreads();
      if (tid == 0) {
        tc_fence_after();
        const uint64_t da = make_smem_desc(smem_u32(sm.p[kc]), 128), db = make_smem_desc(smem_u32(vt), 128);
#pragma unroll
        for (int kk = 0; kk < kAttChunk / 16; ++kk)
          tc_mma_bf16(tO, da + 2ull * kk, db + 2ull * kk, make_idesc_bf16(kAttHeads, kAttHalf),
                      (kc > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&sm.pv_done[st]);
      }
      ++pv_issued[st];
#pragma unroll
      for (int i = 0; i < 8; ++i) xa[i] = xb[i];
    }
    const int last_pv = (kAttPvChunks - 1) & 1;
    if (ok) ok = mbar_wait(&sm.pv_done[last_pv], (pv_issued[last_pv] - 1) & 1u, ctl, DETAIL_WAIT_ACCFULL);
    ok = !__syncthreads_or(!ok);
    if (ok && warp < 4) {
      tc_fence_after();
      const uint32_t h = warp * 32u + lane;
      const uint32_t lane_base = (warp * 32u) << 16;
      float* dst = p.o_part + ((static_cast<size_t>(b) * n_split + c) * kAttHeads + h) * kAttDv + v * kAttHalf;
      for (int cc = 0; cc < kAttHalf / 32; ++cc) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tO + lane_base + cc * 32, r);
        tmem_wait_ld_regs(r);
#pragma unroll
        for (int j = 0; j < 32; j += 4)
          *reinterpret_cast<float4*>(dst + cc * 32 + j) =
              make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]), __uint_as_float(r[j + 2]),
                          __uint_as_float(r[j + 3]));
      }
      if (v == 0) {
        float* ml = p.ml + (static_cast<size_t>(b) * n_split + c) * 2 * kAttHeads;
        ml[h] = sm.m[h];
        ml[kAttHeads + h] = sm.l[h];
      }
      tc_fence_before();
    }
    __syncthreads();  // O is read before the next half's MMAs overwrite it
  }
  if (!ok && tid == 0) {
    // Let the MMAs this CTA issued land before its TMEM is freed (bounded).
    for (int i = 0; i < kAttQkStages; ++i)
      if (qk_issued[i]) mbar_wait_drain(&sm.qk_done[i], (qk_issued[i] - 1) & 1u, p.budget_ns);
    for (int i = 0; i < 2; ++i)
      if (pv_issued[i]) mbar_wait_drain(&sm.pv_done[i], (pv_issued[i] - 1) & 1u, p.budget_ns);
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// out[b][h][d] = sum_c e^(m_c - M) O_c[h][d] / sum_c e^(m_c - M) l_c over the request's splits
// (M the largest m_c); a head whose splits selected nothing gets zeros.
__global__ void __launch_bounds__(128) attention_combine_kernel(const float* __restrict__ o_part,
                                                                const float* __restrict__ ml, int n_split,
                                                                float scale_log2, float* __restrict__ out) {
  const int h = blockIdx.x, b = blockIdx.y;
  float M = -INFINITY;
  for (int c = 0; c < n_split; ++c)
    M = fmaxf(M, ml[(static_cast<size_t>(b) * n_split + c) * 2 * kAttHeads + h]);
  float wsum = 0.0f;
  float w[DSA_MAX_TOPK / kAttSplit];
  for (int c = 0; c < n_split; ++c) {
    const float* mlc = ml + (static_cast<size_t>(b) * n_split + c) * 2 * kAttHeads;
    const float mc = mlc[h];
    w[c] = (mc == -INFINITY) ? 0.0f : exp2f((mc - M) * scale_log2);
    wsum += w[c] * mlc[kAttHeads + h];
  }
  const float inv = wsum > 0.0f ? 1.0f / wsum : 0.0f;
  for (int d = threadIdx.x; d < kAttDv; d += 128) {
    float acc = 0.0f;
    for (int c = 0; c < n_split; ++c)
      acc += w[c] * o_part[((static_cast<size_t>(b) * n_split + c) * kAttHeads + h) * kAttDv + d];
    out[(static_cast<size_t>(b) * kAttHeads + h) * kAttDv + d] = acc * inv;
  }
}

size_t attention_workspace_bytes(int B, int topk) {
  const size_t n_split = static_cast<size_t>(topk) / kAttSplit;
  const size_t o = static_cast<size_t>(B) * n_split * kAttHeads * kAttDv * sizeof(float);
  const size_t ml = static_cast<size_t>(B) * n_split * 2 * kAttHeads * sizeof(float);
  return DSA_WS_HEADER_BYTES + o + ml;
}

dsa_status launch_attention(const AttentionLaunch& a) {
  const int n_split = a.topk / kAttSplit;
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
  attention_combine_kernel<<<dim3(kAttHeads, a.B), 128, 0, a.stream>>>(p.o_part, p.ml, n_split,
                                                                        p.scale_log2, a.out);
  return cuda_status(cudaGetLastError());
}

}  // namespace dsa

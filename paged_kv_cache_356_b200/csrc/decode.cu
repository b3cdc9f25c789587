// pa_decode: one decode step of scaled dot-product attention over the paged
// KV cache, with the block-table translation inside the inner loop, a
// split-context partition of PA_PARTITION_TOKENS tokens, and a log-sum-exp
// merge of the partitions.
//
// PagedAttention Internals, "3. Fused PagedAttention CUDA Kernel": the kernel
// walks the block table in its inner attention loop, fetches the scattered
// K/V pages into shared memory and runs scaled dot-product attention.
// What is PagedAttention?, "On-the-Fly CUDA Block Fetching".
//
// Work decomposition: one CTA per (sequence b, kv head, partition p).  Every
// K/V byte of a sequence is read exactly once; the CTA serves all G query
// heads that share the kv head (GQA), so a page is never fetched twice.
//
// Two partition kernels produce identical partials:
//   decode_tc_kernel   (bf16/f16, head_dim 64/128/256, G <= 8, block_size a
//                      multiple of 16): each warp streams 16-token tiles of K
//                      and V through a cp.async multi-stage pipeline into
//                      XOR-swizzled shared memory and runs both contractions
//                      on the tensor cores with mma.sync m16n8k16:
//                        S^T[16 tok x 8 heads] = K_tile[16 x D] . Q^T[D x 8]
//                        O^T[D x 8 heads]     += V_tile^T[D x 16] . P^T[16 x 8]
//                      (tokens on M, the GQA group on N -- no padded rows);
//                      P^T is re-laid out between the two with movmatrix and
//                      fed as a 16-bit high part plus its rounding residual.
//   decode_cc_kernel   (any dtype incl. fp32, any block size): CUDA cores, one
//                      token per warp step, lanes split head_dim.
// Both keep an online softmax (running max m, running sum l, fp32) per head,
// merge their warps through shared memory, and write either the final output
// (one partition) or the partition's (o_p / l_p, m_p, l_p).  decode_reduce
// then merges partitions: M = max m_p, w_p = l_p e^(m_p - M),
// out = sum w_p o_p / sum w_p.
//
// pa_decode_shared_prefix computes the same result, but a whole partition that
// a group of sequences shares (the same physical pages: forked beams, a common
// prompt) is read once for the whole group by a joint kernel serving up to
// PA_PREFIX_QUERIES_PER_CTA queries -- a dense contraction on the
// fifth-generation tensor cores.  The default joint kernel is the balanced one
// (decode_shared_seg_kernel): equal ranges of 64-token steps per SM over the
// shared partitions, with the members' own tokens folded in or left to the
// per-sequence kernel; a merge follows.  pa_decode_verify treats a sequence's T
// draft tokens as such a group over its own context, each row masked at its
// own causal limit.
#include <math.h>

#include <algorithm>
#include <climits>
#include <cstring>
#include <atomic>
#include <type_traits>
#include <mutex>

#include <cuda.h>
#include <cudaTypedefs.h>

#include "device.cuh"
#include "pa_internal.h"
#include "tcgen05.cuh"

namespace pa {
namespace {

constexpr int kPartition = PA_PARTITION_TOKENS;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr unsigned kFull = 0xffffffffu;

struct DecodeArgs {
  const void* q;
  const void* key_cache;
  const void* value_cache;
  const int32_t* block_tables;
  const int32_t* context_lens;
  void* out;
  float* o_part;
  float* m_part;
  float* l_part;
  int32_t* status;
  const int32_t* first_partition;  // optional: partitions [0, first) of b come from the shared-prefix kernel
  int skip_members;                // with first_partition: sequences with first > 0 are left out entirely
  int partition_base;              // grid z of the partition kernels starts at this partition
  int wait_first;                  // tensor-core kernel launched as a programmatic dependent: wait for the
                                   // grid before it ahead of the first read
  int max_blocks_per_seq;
  int num_q_heads;
  int num_kv_heads;
  int group;
  int block_size;
  int num_blocks;
  int max_partitions;
  float qk_scale_log2;  // softmax scale * log2(e): scores are kept in base 2
};

// Context length of sequence b, clamped to what its table can address.
__device__ __forceinline__ int context_of(const DecodeArgs& a, int b, bool report) {
  int ctx = __ldg(a.context_lens + b);
  const int cap = a.max_blocks_per_seq * a.block_size;
  if (ctx < 0 || ctx > cap) {
    if (report) flag_status(a.status, PA_DEV_BAD_CTX);
    ctx = ctx < 0 ? 0 : cap;
  }
  return ctx;
}

// Merge per-warp (m, l, o) held in shared memory and store the CTA's result
// for heads [h0, h0 + nh): the final row if the sequence has one partition,
// else the partition's partials.  o_w is [warps][heads_stride][D].
template <typename T, int D>
__device__ __forceinline__ void merge_and_store(const DecodeArgs& a, int b, int h0, int nh, int p, int np,
                                                int warps, int heads_stride, const float* o_w, const float* m_w,
                                                const float* l_w) {
  for (int i = threadIdx.x; i < nh * D; i += blockDim.x) {
    const int j = i / D;
    const int d = i - j * D;
    float mx = -INFINITY;
    for (int w = 0; w < warps; ++w) mx = fmaxf(mx, m_w[w * heads_stride + j]);
    float l = 0.f, o = 0.f;
    if (mx != -INFINITY) {
      for (int w = 0; w < warps; ++w) {
        const float c = exp2f(m_w[w * heads_stride + j] - mx);
        l += l_w[w * heads_stride + j] * c;
        o += o_w[((size_t)w * heads_stride + j) * D + d] * c;
      }
    }
    const float res = l > 0.f ? o / l : 0.f;
    const int64_t row = (int64_t)b * a.num_q_heads + h0 + j;
    if (np <= 1) {
      reinterpret_cast<T*>(a.out)[row * D + d] = from_float<T>(res);
    } else {
      const int64_t part = row * a.max_partitions + p;
      a.o_part[part * D + d] = res;
      if (d == 0) {
        a.m_part[part] = mx == -INFINITY ? -INFINITY : mx * kLn2;
        a.l_part[part] = l;
      }
    }
  }
}

template <typename T, int D>
__device__ __forceinline__ void store_zero_rows(const DecodeArgs& a, int b, int h0, int nh) {
  T* out = reinterpret_cast<T*>(a.out);
  for (int i = threadIdx.x; i < nh * D; i += blockDim.x)
    out[((int64_t)b * a.num_q_heads + h0) * D + i] = from_float<T>(0.f);
}

// A partition kernel launched as a programmatic dependent of the shared-prefix
// kernel (so that its CTAs fill the SMs that kernel's last wave leaves idle)
// must still finish after it, for the merge that follows: one thread waits for
// the prerequisite grid on the way out.  On an ordinary launch the wait returns
// at once.
struct AfterPrerequisiteGrid {
  bool on;
  __device__ ~AfterPrerequisiteGrid() {
    if (on) asm volatile("griddepcontrol.wait;\n" ::: "memory");
  }
};

// ---------------------------------------------------------------------------
// CUDA-core partition kernel.  Grid (num_seqs, num_kv_heads * head_chunks, P);
// a CTA serves up to GC query heads of one kv head.
// ---------------------------------------------------------------------------
template <typename T, int D, int GC, int NW>
__global__ void __launch_bounds__(NW * 32) decode_cc_kernel(const DecodeArgs a) {
  const AfterPrerequisiteGrid after{threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0};
  // A joint kernel launched after this one as a programmatic dependent may start now.
  if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  constexpr int VPL = D / 32;
  __shared__ float o_w[NW * GC * D];
  __shared__ float m_w[NW * GC];
  __shared__ float l_w[NW * GC];

  const int b = blockIdx.x;
  const int chunks = (a.group + GC - 1) / GC;
  const int kvh = blockIdx.y / chunks;
  const int chunk = blockIdx.y - kvh * chunks;
  const int h0 = kvh * a.group + chunk * GC;
  const int nh = min(GC, a.group - chunk * GC);
  const int p = blockIdx.z + a.partition_base;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int ctx = context_of(a, b, threadIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0);
  const int np = (ctx + kPartition - 1) / kPartition;
  if (p >= max(np, 1)) return;
  if (a.first_partition && (a.skip_members ? __ldg(a.first_partition + b) > 0 : p < __ldg(a.first_partition + b)))
    return;
  if (ctx == 0) {
    store_zero_rows<T, D>(a, b, h0, nh);
    return;
  }
  const int tok_begin = p * kPartition;
  const int tok_end = min(ctx, tok_begin + kPartition);

  float qv[GC][VPL];
#pragma unroll
  for (int g = 0; g < GC; ++g) {
    if (g < nh) {
      load_floats<T, VPL>(reinterpret_cast<const T*>(a.q) + ((int64_t)b * a.num_q_heads + h0 + g) * D + lane * VPL,
                          qv[g]);
#pragma unroll
      for (int i = 0; i < VPL; ++i) qv[g][i] *= a.qk_scale_log2;
    } else {
#pragma unroll
      for (int i = 0; i < VPL; ++i) qv[g][i] = 0.f;
    }
  }
  float m[GC], l[GC], o[GC][VPL];
#pragma unroll
  for (int g = 0; g < GC; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) o[g][i] = 0.f;
  }

  const T* kc = reinterpret_cast<const T*>(a.key_cache);
  const T* vc = reinterpret_cast<const T*>(a.value_cache);
  const int32_t* table = a.block_tables + (int64_t)b * a.max_blocks_per_seq;
  for (int tok = tok_begin + warp; tok < tok_end; tok += NW) {
    const int page = __ldg(table + tok / a.block_size);
    if ((unsigned)page >= (unsigned)a.num_blocks) {
      if (lane == 0) flag_status(a.status, PA_DEV_BAD_PAGE);
      continue;
    }
    const int64_t row =
        (((int64_t)page * a.num_kv_heads + kvh) * a.block_size + tok % a.block_size) * D + lane * VPL;
    float kf[VPL], vf[VPL];
    load_floats<T, VPL>(kc + row, kf);
    load_floats<T, VPL>(vc + row, vf);
    float s[GC];
#pragma unroll
    for (int g = 0; g < GC; ++g) {
      float acc = 0.f;
#pragma unroll
      for (int i = 0; i < VPL; ++i) acc = fmaf(qv[g][i], kf[i], acc);
      s[g] = acc;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
#pragma unroll
      for (int g = 0; g < GC; ++g) s[g] += __shfl_xor_sync(kFull, s[g], off);
    }
#pragma unroll
    for (int g = 0; g < GC; ++g) {
      const float mn = fmaxf(m[g], s[g]);
      const float alpha = exp2f(m[g] - mn);
      const float pr = exp2f(s[g] - mn);
      l[g] = l[g] * alpha + pr;
#pragma unroll
      for (int i = 0; i < VPL; ++i) o[g][i] = fmaf(pr, vf[i], o[g][i] * alpha);
      m[g] = mn;
    }
  }

#pragma unroll
  for (int g = 0; g < GC; ++g) {
#pragma unroll
    for (int i = 0; i < VPL; ++i) o_w[(warp * GC + g) * D + lane * VPL + i] = o[g][i];
    if (lane == 0) {
      m_w[warp * GC + g] = m[g];
      l_w[warp * GC + g] = l[g];
    }
  }
  __syncthreads();
  merge_and_store<T, D>(a, b, h0, nh, p, np, NW, GC, o_w, m_w, l_w);
}

// ---------------------------------------------------------------------------
// Tensor-core partition kernel.  Grid (num_seqs, num_kv_heads, P); NW warps,
// each streaming its own contiguous run of 16-token tiles of the partition
// through STAGES shared-memory buffers.
//
// Shared memory per warp and stage: K tile then V tile, [16 rows][D] 16-bit,
// rows of 2*D bytes; 16-byte chunk c of row r is stored at chunk c ^ (r & 7),
// so the 8 row addresses of every ldmatrix phase hit 8 distinct bank groups.
// ---------------------------------------------------------------------------
template <int D, int NW, int STAGES>
struct TcShape {
  static constexpr int kRowBytes = 2 * D;
  static constexpr int kChunksPerRow = kRowBytes / 16;
  static constexpr int kTile = 16;
  static constexpr int kTileBytes = kTile * kRowBytes;
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kWarpBytes = STAGES * kStageBytes;
  static constexpr int kSmemBytes = NW * kWarpBytes;
  static constexpr int kChunksPerLane = kTile * kChunksPerRow / 32;
  static_assert(8 * D * 4 + 16 * 4 <= kWarpBytes, "warp region must hold its merge scratch");
};

template <typename T, int D, int NW, int STAGES>
__global__ void __launch_bounds__(NW * 32) decode_tc_kernel(const DecodeArgs a) {
  const AfterPrerequisiteGrid after{threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0};
  // A joint kernel launched after this one as a programmatic dependent may start now.
  if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  // Launched early after the step's cache write: nothing is read before that grid is done.
  if (a.wait_first) asm volatile("griddepcontrol.wait;\n" ::: "memory");
  using S = TcShape<D, NW, STAGES>;
  constexpr int KSTEPS = D / 16;
  constexpr int MTILES = D / 16;
  extern __shared__ __align__(128) uint8_t smem[];

  const int b = blockIdx.x;
  const int kvh = blockIdx.y;
  const int p = blockIdx.z + a.partition_base;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2;  // fragment row group
  const int t = lane & 3;   // fragment column pair
  const int G = a.group;
  const int h0 = kvh * G;

  const int ctx = context_of(a, b, threadIdx.x == 0 && kvh == 0 && blockIdx.z == 0);
  const int np = (ctx + kPartition - 1) / kPartition;
  if (p >= max(np, 1)) return;
  if (a.first_partition && (a.skip_members ? __ldg(a.first_partition + b) > 0 : p < __ldg(a.first_partition + b)))
    return;
  if (ctx == 0) {
    store_zero_rows<T, D>(a, b, h0, G);
    return;
  }
  const int bs = a.block_size;
  const int tok_begin = p * kPartition;
  const int tok_end = min(ctx, tok_begin + kPartition);
  const int ntiles = (tok_end - tok_begin + S::kTile - 1) / S::kTile;
  const int per_warp = (ntiles + NW - 1) / NW;
  const int first_tile = warp * per_warp;
  const int my_tiles = max(0, min(per_warp, ntiles - first_tile));

  // This partition's block-table entries, one per lane (at most 32 since
  // block_size >= 16); every tile's page is then a register shuffle away.
  const int first_block = tok_begin / bs;
  const int nblk = (tok_end - 1) / bs - first_block + 1;
  int lane_page = 0;
  if (lane < nblk) lane_page = __ldg(a.block_tables + (int64_t)b * a.max_blocks_per_seq + first_block + lane);

  // Q^T fragments (B operand, k = head_dim, n = query head of the group).
  uint32_t qf[KSTEPS][2];
  {
    const bool real = g < G;
    const uint32_t* qrow = reinterpret_cast<const uint32_t*>(reinterpret_cast<const T*>(a.q) +
                                                             ((int64_t)b * a.num_q_heads + h0 + (real ? g : 0)) * D);
#pragma unroll
    for (int ks = 0; ks < KSTEPS; ++ks) {
      qf[ks][0] = real ? __ldg(qrow + 8 * ks + t) : 0u;
      qf[ks][1] = real ? __ldg(qrow + 8 * ks + 4 + t) : 0u;
    }
  }

  uint8_t* wsm = smem + warp * S::kWarpBytes;
  const uint32_t wsm_u32 = smem_u32(wsm);
  const T* kc = reinterpret_cast<const T*>(a.key_cache);
  const T* vc = reinterpret_cast<const T*>(a.value_cache);

  // Issue the cp.async copies of local tile i into stage `stage`.
  auto load_tile = [&](int i, int stage) {
    const int tok0 = tok_begin + (first_tile + i) * S::kTile;
    int valid = min(S::kTile, tok_end - tok0);
    int page = __shfl_sync(kFull, lane_page, tok0 / bs - first_block);
    if ((unsigned)page >= (unsigned)a.num_blocks) {
      if (lane == 0) flag_status(a.status, PA_DEV_BAD_PAGE);
      valid = 0;
      page = 0;
    }
    const int64_t row0 = ((int64_t)page * a.num_kv_heads + kvh) * bs + (tok0 % bs);
    const T* ksrc = kc + row0 * D;
    const T* vsrc = vc + row0 * D;
    const uint32_t kdst = wsm_u32 + stage * S::kStageBytes;
    const uint32_t vdst = kdst + S::kTileBytes;
#pragma unroll
    for (int j = 0; j < S::kChunksPerLane; ++j) {
      const int idx = lane + 32 * j;
      const int r = idx / S::kChunksPerRow;
      const int c = idx - r * S::kChunksPerRow;
      const bool ok = r < valid;
      const int64_t src = (int64_t)(ok ? r : 0) * D + c * 8;
      const uint32_t dst = r * S::kRowBytes + ((c ^ (r & 7)) << 4);
      cp_async_16(kdst + dst, ksrc + src, ok ? 16u : 0u);
      cp_async_16(vdst + dst, vsrc + src, ok ? 16u : 0u);
    }
    return valid;
  };

  float o[MTILES][4];
#pragma unroll
  for (int mt = 0; mt < MTILES; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
  float m[2] = {-INFINITY, -INFINITY};  // heads 2t, 2t+1 (base-2 scores)
  float l[2] = {0.f, 0.f};              // this lane's tokens only; reduced at the end

#pragma unroll
  for (int i = 0; i < STAGES - 1; ++i) {
    if (i < my_tiles) load_tile(i, i);
    cp_async_commit();
  }

  for (int i = 0; i < my_tiles; ++i) {
    {
      const int nxt = i + STAGES - 1;
      if (nxt < my_tiles) load_tile(nxt, nxt % STAGES);
      cp_async_commit();
    }
    cp_async_wait<STAGES - 1>();
    __syncwarp();

    const int stage = i % STAGES;
    const uint32_t kbase = wsm_u32 + stage * S::kStageBytes;
    const uint32_t vbase = kbase + S::kTileBytes;
    const int tok0 = tok_begin + (first_tile + i) * S::kTile;
    int valid = min(S::kTile, tok_end - tok0);
    {
      const int page = __shfl_sync(kFull, lane_page, tok0 / bs - first_block);
      if ((unsigned)page >= (unsigned)a.num_blocks) valid = 0;
    }

    // S^T = K_tile . Q^T : two accumulator chains over the head_dim k-steps.
    float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
    {
      const int r = (lane & 7) + ((lane >> 3) & 1) * 8;
      const uint32_t rbase = kbase + r * S::kRowBytes;
#pragma unroll
      for (int ks = 0; ks < KSTEPS; ++ks) {
        const int c = 2 * ks + (lane >> 4);
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4(rbase + ((c ^ (r & 7)) << 4), a0, a1, a2, a3);
        if (ks & 1)
          mma_16816<T>(s1, a0, a1, a2, a3, qf[ks][0], qf[ks][1]);
        else
          mma_16816<T>(s0, a0, a1, a2, a3, qf[ks][0], qf[ks][1]);
      }
    }
    // s[0], s[1]: token g, heads 2t, 2t+1; s[2], s[3]: token g + 8.
    float s[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) s[e] = (s0[e] + s1[e]) * a.qk_scale_log2;
    if (g >= valid) s[0] = s[1] = -INFINITY;
    if (g + 8 >= valid) s[2] = s[3] = -INFINITY;

    float pr[4], alpha[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      float mx = fmaxf(s[j], s[2 + j]);
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 16));
      const float mn = fmaxf(m[j], mx);
      const float base = mn == -INFINITY ? 0.f : mn;
      alpha[j] = exp2f(m[j] - base);
      pr[j] = exp2f(s[j] - base);
      pr[2 + j] = exp2f(s[2 + j] - base);
      l[j] = l[j] * alpha[j] + pr[j] + pr[2 + j];
      m[j] = mn;
    }
#pragma unroll
    for (int mt = 0; mt < MTILES; ++mt) {
      o[mt][0] *= alpha[0];
      o[mt][1] *= alpha[1];
      o[mt][2] *= alpha[0];
      o[mt][3] *= alpha[1];
    }
    // P^T as the B operand (k = token, n = head), split into a 16-bit high
    // part and the 16-bit rounding residual (P = P_hi + P_lo to ~2^-17), so
    // the weights lose nothing to the 16-bit operand format; each 8x8 half is
    // transposed into the B layout with movmatrix.
    const uint32_t hi0 = pack2<T>(pr[0], pr[1]);
    const uint32_t hi1 = pack2<T>(pr[2], pr[3]);
    const float2 r0 = unpack2<T>(hi0), r1 = unpack2<T>(hi1);
    const uint32_t lo0 = pack2<T>(pr[0] - r0.x, pr[1] - r0.y);
    const uint32_t lo1 = pack2<T>(pr[2] - r1.x, pr[3] - r1.y);
    const uint32_t pb0 = movmatrix_trans(hi0), pb1 = movmatrix_trans(hi1);
    const uint32_t pl0 = movmatrix_trans(lo0), pl1 = movmatrix_trans(lo1);

    // O^T += V_tile^T . (P_hi^T + P_lo^T), one m16 tile of head_dim at a time.
    {
      const int mat = lane >> 3;
      const int r = (lane & 7) + ((mat >> 1) << 3);
      const uint32_t rbase = vbase + r * S::kRowBytes;
#pragma unroll
      for (int mt = 0; mt < MTILES; ++mt) {
        const int c = 2 * mt + (mat & 1);
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4_trans(rbase + ((c ^ (r & 7)) << 4), a0, a1, a2, a3);
        mma_16816<T>(o[mt], a0, a1, a2, a3, pb0, pb1);
        mma_16816<T>(o[mt], a0, a1, a2, a3, pl0, pl1);
      }
    }
    __syncwarp();
  }
  cp_async_wait<0>();
  __syncwarp();

#pragma unroll
  for (int j = 0; j < 2; ++j) {
    l[j] += __shfl_xor_sync(kFull, l[j], 4);
    l[j] += __shfl_xor_sync(kFull, l[j], 8);
    l[j] += __shfl_xor_sync(kFull, l[j], 16);
  }
  // Warp partials into this warp's own region: o[8][D], then m[8], l[8].
  float* o_w = reinterpret_cast<float*>(wsm);
  float* ml_w = o_w + 8 * D;
#pragma unroll
  for (int mt = 0; mt < MTILES; ++mt) {
    const int d = 16 * mt + g;
    o_w[(2 * t) * D + d] = o[mt][0];
    o_w[(2 * t + 1) * D + d] = o[mt][1];
    o_w[(2 * t) * D + d + 8] = o[mt][2];
    o_w[(2 * t + 1) * D + d + 8] = o[mt][3];
  }
  if (g == 0) {
    ml_w[2 * t] = m[0];
    ml_w[2 * t + 1] = m[1];
    ml_w[8 + 2 * t] = l[0];
    ml_w[8 + 2 * t + 1] = l[1];
  }
  __syncthreads();

  // Merge the warps: each region is kWarpBytes apart.
  constexpr int kStrideF = S::kWarpBytes / 4;
  const float* base_f = reinterpret_cast<const float*>(smem);
  for (int i = threadIdx.x; i < G * D; i += NW * 32) {
    const int j = i / D;
    const int d = i - j * D;
    float mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) mx = fmaxf(mx, base_f[w * kStrideF + 8 * D + j]);
    float lsum = 0.f, osum = 0.f;
    if (mx != -INFINITY) {
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        const float c = exp2f(base_f[w * kStrideF + 8 * D + j] - mx);
        lsum += base_f[w * kStrideF + 8 * D + 8 + j] * c;
        osum += base_f[w * kStrideF + j * D + d] * c;
      }
    }
    const float res = lsum > 0.f ? osum / lsum : 0.f;
    const int64_t row = (int64_t)b * a.num_q_heads + h0 + j;
    if (np <= 1) {
      reinterpret_cast<T*>(a.out)[row * D + d] = from_float<T>(res);
    } else {
      const int64_t part = row * a.max_partitions + p;
      a.o_part[part * D + d] = res;
      if (d == 0) {
        a.m_part[part] = mx == -INFINITY ? -INFINITY : mx * kLn2;
        a.l_part[part] = lsum;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Shared-prefix partition kernel on mma.sync (the fallback of the tcgen05
// kernel below).  Grid (chunk, kv head, shared partition); 8 warps.  A chunk
// is up to 128 queries: `count` member sequences x G query
// heads of one kv head, all reading the same 512-token partition through the
// leader's table.  The CTA streams the partition's 16-token K/V tiles once
// through a CTA-wide cp.async pipeline (STAGES buffers, every thread copies
// its share); warp w owns queries [16w, 16w + 16) as two 8-wide MMA n-tiles:
//   S^T[16 tok x 16 q] = K_tile . Q^T,   O^T[D x 16 q] += V_tile^T . P^T
// with the same swizzle and online softmax as the per-sequence kernel (P as
// a 16-bit operand; the residual MMA is a template option).  Each warp writes
// its queries' partition partials.
// ---------------------------------------------------------------------------
template <int D, int STAGES>
struct SharedShape {
  static constexpr int kWarps = PA_PREFIX_QUERIES_PER_CTA / 16;
  static constexpr int kThreads = 32 * kWarps;
  static constexpr int kRowBytes = 2 * D;
  static constexpr int kChunksPerRow = kRowBytes / 16;
  static constexpr int kTile = 16;
  static constexpr int kTiles = kPartition / kTile;
  static constexpr int kTileBytes = kTile * kRowBytes;
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kSmemBytes = STAGES * kStageBytes;
  static constexpr int kCopiesPerThread = 2 * kTile * kChunksPerRow / kThreads;
  static_assert(2 * kTile * kChunksPerRow % kThreads == 0, "tile copies must split evenly");
};

template <typename T, int D, int STAGES, bool RESIDUAL>
__global__ void __launch_bounds__(PA_PREFIX_QUERIES_PER_CTA * 2, 2) decode_shared_kernel(const DecodeArgs a, const int32_t* __restrict__ chunks,
                                                            const int32_t* __restrict__ members, int num_members,
                                                            int num_seqs) {
  using S = SharedShape<D, STAGES>;
  constexpr int KSTEPS = D / 16;
  constexpr int MTILES = D / 16;
  constexpr int NT = 2;  // 8-query n-tiles per warp
  extern __shared__ __align__(128) uint8_t smem[];

  const int c = blockIdx.x;
  const int kvh = blockIdx.y;
  const int p = blockIdx.z;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2;
  const int t = lane & 3;
  const int leader = __ldg(chunks + 4 * c);
  const int moff = __ldg(chunks + 4 * c + 1);
  const int mcount = __ldg(chunks + 4 * c + 2);
  const int sp = __ldg(chunks + 4 * c + 3);
  if (p >= sp) return;
  const int bs = a.block_size;
  const int G = a.group;
  const int tok_begin = p * kPartition;
  if ((unsigned)leader >= (unsigned)num_seqs || moff < 0 || mcount < 0 || (int64_t)moff + mcount > num_members ||
      (int64_t)tok_begin + kPartition > (int64_t)a.max_blocks_per_seq * bs || p >= a.max_partitions) {
    if (threadIdx.x == 0) flag_status(a.status, PA_DEV_BAD_PLAN);
    return;
  }
  const int first_block = tok_begin / bs;
  const int nblk = (tok_begin + kPartition - 1) / bs - first_block + 1;  // <= 32 for bs >= 16
  int lane_page = 0;
  if (lane < nblk) lane_page = __ldg(a.block_tables + (int64_t)leader * a.max_blocks_per_seq + first_block + lane);

  // Query of column n of this warp's n-tile nt: member (16w + 8nt + n) / G, head (.) % G.
  auto query_row = [&](int qi) -> int64_t {  // row of q / out for query qi, or -1
    const int mi = qi / G;
    if (mi >= mcount) return -1;
    const int b = __ldg(members + moff + mi);
    if ((unsigned)b >= (unsigned)num_seqs) return -1;
    return (int64_t)b * a.num_q_heads + kvh * G + (qi - mi * G);
  };

  uint32_t qf[NT][KSTEPS][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int64_t row = query_row(warp * 16 + nt * 8 + g);
    const uint32_t* qrow =
        reinterpret_cast<const uint32_t*>(reinterpret_cast<const T*>(a.q) + (row < 0 ? 0 : row) * D);
#pragma unroll
    for (int ks = 0; ks < KSTEPS; ++ks) {
      qf[nt][ks][0] = row >= 0 ? __ldg(qrow + 8 * ks + t) : 0u;
      qf[nt][ks][1] = row >= 0 ? __ldg(qrow + 8 * ks + 4 + t) : 0u;
    }
  }
  const bool warp_busy = (warp * 16) / G < mcount;

  const uint32_t smem_base = smem_u32(smem);
  const T* kc = reinterpret_cast<const T*>(a.key_cache);
  const T* vc = reinterpret_cast<const T*>(a.value_cache);
  // Every thread copies kCopiesPerThread 16-byte chunks of tile i (K chunks, then V chunks).
  auto load_tile = [&](int i, int stage) {
    const int tok0 = tok_begin + i * S::kTile;
    int page = __shfl_sync(kFull, lane_page, tok0 / bs - first_block);
    bool ok = (unsigned)page < (unsigned)a.num_blocks;
    if (!ok) {
      if (threadIdx.x == 0) flag_status(a.status, PA_DEV_BAD_PAGE);
      page = 0;
    }
    const int64_t row0 = ((int64_t)page * a.num_kv_heads + kvh) * bs + (tok0 % bs);
    const uint32_t kdst = smem_base + stage * S::kStageBytes;
#pragma unroll
    for (int j = 0; j < S::kCopiesPerThread; ++j) {
      const int idx = threadIdx.x + S::kThreads * j;
      const int half = idx / (S::kTile * S::kChunksPerRow);  // 0: K, 1: V
      const int rem = idx - half * (S::kTile * S::kChunksPerRow);
      const int r = rem / S::kChunksPerRow;
      const int cc = rem - r * S::kChunksPerRow;
      const T* src = (half ? vc : kc) + (row0 + r) * D + cc * 8;
      const uint32_t dst = kdst + half * S::kTileBytes + r * S::kRowBytes + ((cc ^ (r & 7)) << 4);
      cp_async_16(dst, src, ok ? 16u : 0u);
    }
  };

  float o[MTILES][NT][4];
#pragma unroll
  for (int mt = 0; mt < MTILES; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) o[mt][nt][0] = o[mt][nt][1] = o[mt][nt][2] = o[mt][nt][3] = 0.f;
  float m[NT][2], l[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) m[nt][0] = m[nt][1] = -INFINITY, l[nt][0] = l[nt][1] = 0.f;

#pragma unroll
  for (int i = 0; i < STAGES - 1; ++i) {
    load_tile(i, i);
    cp_async_commit();
  }
  for (int i = 0; i < S::kTiles; ++i) {
    {
      const int nxt = i + STAGES - 1;
      if (nxt < S::kTiles) load_tile(nxt, nxt % STAGES);
      cp_async_commit();
    }
    cp_async_wait<STAGES - 1>();
    __syncthreads();
    if (warp_busy) {
      const int stage = i % STAGES;
      const uint32_t kbase = smem_base + stage * S::kStageBytes;
      const uint32_t vbase = kbase + S::kTileBytes;
      const int tok0 = tok_begin + i * S::kTile;
      const bool valid = (unsigned)__shfl_sync(kFull, lane_page, tok0 / bs - first_block) < (unsigned)a.num_blocks;

      float sacc[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
      {
        const int r = (lane & 7) + ((lane >> 3) & 1) * 8;
        const uint32_t rbase = kbase + r * S::kRowBytes;
#pragma unroll
        for (int ks = 0; ks < KSTEPS; ++ks) {
          const int cc = 2 * ks + (lane >> 4);
          uint32_t a0, a1, a2, a3;
          ldmatrix_x4(rbase + ((cc ^ (r & 7)) << 4), a0, a1, a2, a3);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) mma_16816<T>(sacc[nt], a0, a1, a2, a3, qf[nt][ks][0], qf[nt][ks][1]);
        }
      }
      uint32_t pb[NT][2], pl[NT][2];
      float alpha[NT][2];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        float sv[4], pr[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) sv[e] = valid ? sacc[nt][e] * a.qk_scale_log2 : -INFINITY;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          float mx = fmaxf(sv[j], sv[2 + j]);
          mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 4));
          mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 8));
          mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 16));
          const float mn = fmaxf(m[nt][j], mx);
          const float base = mn == -INFINITY ? 0.f : mn;
          alpha[nt][j] = exp2f(m[nt][j] - base);
          pr[j] = exp2f(sv[j] - base);
          pr[2 + j] = exp2f(sv[2 + j] - base);
          l[nt][j] = l[nt][j] * alpha[nt][j] + pr[j] + pr[2 + j];
          m[nt][j] = mn;
        }
        const uint32_t hi0 = pack2<T>(pr[0], pr[1]);
        const uint32_t hi1 = pack2<T>(pr[2], pr[3]);
        const float2 r0 = unpack2<T>(hi0), r1 = unpack2<T>(hi1);
        pb[nt][0] = movmatrix_trans(hi0);
        pb[nt][1] = movmatrix_trans(hi1);
        if constexpr (RESIDUAL) {
          pl[nt][0] = movmatrix_trans(pack2<T>(pr[0] - r0.x, pr[1] - r0.y));
          pl[nt][1] = movmatrix_trans(pack2<T>(pr[2] - r1.x, pr[3] - r1.y));
        } else {
          (void)r0;
          (void)r1;
          pl[nt][0] = pl[nt][1] = 0u;
        }
      }
      const int mat = lane >> 3;
      const int r = (lane & 7) + ((mat >> 1) << 3);
      const uint32_t rbase = vbase + r * S::kRowBytes;
#pragma unroll
      for (int mt = 0; mt < MTILES; ++mt) {
        const int cc = 2 * mt + (mat & 1);
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4_trans(rbase + ((cc ^ (r & 7)) << 4), a0, a1, a2, a3);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          o[mt][nt][0] *= alpha[nt][0];
          o[mt][nt][1] *= alpha[nt][1];
          o[mt][nt][2] *= alpha[nt][0];
          o[mt][nt][3] *= alpha[nt][1];
          mma_16816<T>(o[mt][nt], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
          if constexpr (RESIDUAL) mma_16816<T>(o[mt][nt], a0, a1, a2, a3, pl[nt][0], pl[nt][1]);
        }
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();
  if (!warp_busy) return;

  // Partials of this warp's 16 queries: column 2t + j of n-tile nt.
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      float lj = l[nt][j];
      lj += __shfl_xor_sync(kFull, lj, 4);
      lj += __shfl_xor_sync(kFull, lj, 8);
      lj += __shfl_xor_sync(kFull, lj, 16);
      const int64_t row = query_row(warp * 16 + nt * 8 + 2 * t + j);
      if (row < 0) continue;
      const int64_t part = row * a.max_partitions + p;
      const float inv = lj > 0.f ? 1.f / lj : 0.f;
      float* dst = a.o_part + part * D;
#pragma unroll
      for (int mt = 0; mt < MTILES; ++mt) {
        dst[16 * mt + g] = o[mt][nt][j] * inv;
        dst[16 * mt + g + 8] = o[mt][nt][2 + j] * inv;
      }
      if (g == 0) {
        a.m_part[part] = m[nt][j] == -INFINITY ? -INFINITY : m[nt][j] * kLn2;
        a.l_part[part] = lj;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Shared-prefix partition kernel on the 5th-generation tensor cores (tcgen05,
// accumulators in Tensor Memory).  Grid (chunk, kv head, shared partition);
// 4 warps; one CTA serves up to 128 queries (the chunk's members x G heads of
// one kv head, padded with zero rows to the MMA's M = 128) over one shared
// 512-token partition, in 64-token steps:
//   S[128 x 64]  = Q[128 x D] . K_step^T      (tcgen05.mma, A and B from smem)
//   softmax      thread r owns query row r: reads its S row from TMEM, keeps
//                a running max m (rescaling O only when the max grows by more
//                than 2^8, which is exact: O and l share the reference max),
//                writes P as 16-bit values back to TMEM
//   O[128 x D]  += P[128 x 64] . V_step      (tcgen05.mma, A from TMEM)
// Q and the K/V steps are staged by cp.async in the canonical 128-byte-swizzle
// layout (8 rows x 128 B atoms; K and V share the physical layout, K is read
// K-major, V MN-major).  Thread 0 issues the MMAs; tcgen05.commit signals
// mbarriers.  Every wait is bounded: on timeout the CTA flags
// PA_DEV_TIMEOUT, lets its copies land, frees its TMEM and returns.
// ---------------------------------------------------------------------------
template <int D>
struct Tc05Shape {
  static constexpr int kThreads = 128;
  static constexpr int kRows = 128;                       // MMA M: query rows
  static constexpr int kStep = 64;                        // tokens per step: MMA1 N, MMA2 K
  static constexpr int kSteps = kPartition / kStep;       // 8
  static constexpr int kBlocks = D / 64;                  // 64-element swizzle blocks along head_dim
  static constexpr int kQBlockBytes = kRows * 128;        // one 64-wide block of Q
  static constexpr int kQBytes = kBlocks * kQBlockBytes;
  static constexpr int kKVBlockBytes = kStep * 128;       // one 64-wide block of a K or V step
  static constexpr int kTileBytes = kBlocks * kKVBlockBytes;
  static constexpr int kStageBytes = 2 * kTileBytes;      // K then V
  static constexpr int kStages = 2;
  static constexpr int kBarOffset = kQBytes + kStages * kStageBytes;
  static constexpr int kSmemBytes = kBarOffset + 64 + 1024;  // + mbarriers, TMEM address, alignment slack
  static constexpr uint32_t kSCol = 0, kPCol = kStep, kOCol = 128;
  static constexpr uint32_t kTmemCols = 256;
  static_assert(kOCol + D <= kTmemCols, "TMEM columns");
  static_assert(kRows * (D / 8) % kThreads == 0 && 2 * kStep * (D / 8) % kThreads == 0, "copy split");
};

constexpr long long kWaitCycles = 2000000000LL;  // ~1 s at 2 GHz

template <typename T, int D>
__global__ void __launch_bounds__(128, 1) decode_shared_tc05_kernel(const DecodeArgs a, const int32_t* __restrict__ chunks,
                                                                   const int32_t* __restrict__ members,
                                                                   int num_members, int num_seqs) {
  using S = Tc05Shape<D>;
  extern __shared__ uint8_t smem_raw[];
  const int c = blockIdx.x;
  const int kvh = blockIdx.y;
  const int p = blockIdx.z;
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int leader = __ldg(chunks + 4 * c);
  const int moff = __ldg(chunks + 4 * c + 1);
  const int mcount = __ldg(chunks + 4 * c + 2);
  const int sp = __ldg(chunks + 4 * c + 3);
  if (p >= sp) return;
  const int bs = a.block_size;
  const int G = a.group;
  const int tok_begin = p * kPartition;
  if ((unsigned)leader >= (unsigned)num_seqs || moff < 0 || mcount < 0 || (int64_t)moff + mcount > num_members ||
      (int64_t)mcount * G > S::kRows || (int64_t)tok_begin + kPartition > (int64_t)a.max_blocks_per_seq * bs ||
      p >= a.max_partitions) {
    if (tid == 0) flag_status(a.status, PA_DEV_BAD_PLAN);
    return;
  }
  const int nq = mcount * G;  // real query rows
  const int first_block = tok_begin / bs;
  const int nblk = (tok_begin + kPartition - 1) / bs - first_block + 1;  // <= 32 for bs >= 16
  int lane_page = 0;
  if (lane < nblk) lane_page = __ldg(a.block_tables + (int64_t)leader * a.max_blocks_per_seq + first_block + lane);

  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;  // swizzle atoms need 1024-byte alignment
  const uint32_t q_smem = base;
  const uint32_t st_smem = base + S::kQBytes;
  const uint32_t bar_s = base + S::kBarOffset;
  const uint32_t bar_o = bar_s + 8;
  const uint32_t taddr_slot = bar_s + 16;
  uint32_t* taddr_ptr = reinterpret_cast<uint32_t*>(smem_raw + (taddr_slot - raw));

  // Row of q / out for query row r of this chunk, or -1 (padding / bad member).
  auto query_row = [&](int r) -> int64_t {
    if (r >= nq) return -1;
    const int mi = r / G;
    const int b = __ldg(members + moff + mi);
    if ((unsigned)b >= (unsigned)num_seqs) return -1;
    return (int64_t)b * a.num_q_heads + kvh * G + (r - mi * G);
  };

  // -- set-up: mbarriers, TMEM, Q ------------------------------------------------------
  if (tid == 0) {
    tc05::mbar_init(bar_s, 1);
    tc05::mbar_init(bar_o, 1);
    tc05::fence_mbar_init();
  }
  if (warp == 0) {
    tc05::alloc(taddr_slot, S::kTmemCols);
    tc05::relinquish();
  }
  {
    const T* qbase = reinterpret_cast<const T*>(a.q);
#pragma unroll 4
    for (int j = 0; j < S::kRows * (D / 8) / S::kThreads; ++j) {
      const int idx = tid + S::kThreads * j;
      const int r = idx / (D / 8);
      const int ck = idx - r * (D / 8);
      const int64_t row = query_row(r);
      const T* src = qbase + (row < 0 ? 0 : row) * D + ck * 8;
      const uint32_t dst = q_smem + (ck >> 3) * S::kQBlockBytes + r * 128 + (((ck & 7) ^ (r & 7)) << 4);
      cp_async_16(dst, src, row < 0 ? 0u : 16u);
    }
  }
  const T* kc = reinterpret_cast<const T*>(a.key_cache);
  const T* vc = reinterpret_cast<const T*>(a.value_cache);
  // Every thread copies its share of step i's K and V rows into stage `stage`.
  auto load_step = [&](int i, int stage) {
    const uint32_t kdst = st_smem + stage * S::kStageBytes;
#pragma unroll 4
    for (int j = 0; j < 2 * S::kStep * (D / 8) / S::kThreads; ++j) {
      const int idx = tid + S::kThreads * j;
      const int half = idx / (S::kStep * (D / 8));  // 0: K, 1: V
      const int rem = idx - half * (S::kStep * (D / 8));
      const int t = rem / (D / 8);
      const int ck = rem - t * (D / 8);
      const int tok = tok_begin + i * S::kStep + t;
      int page = __shfl_sync(kFull, lane_page, tok / bs - first_block);
      const bool ok = (unsigned)page < (unsigned)a.num_blocks;
      if (!ok) page = 0;
      const T* src = (half ? vc : kc) + (((int64_t)page * a.num_kv_heads + kvh) * bs + tok % bs) * D + ck * 8;
      const uint32_t dst =
          kdst + half * S::kTileBytes + (ck >> 3) * S::kKVBlockBytes + t * 128 + (((ck & 7) ^ (t & 7)) << 4);
      cp_async_16(dst, src, ok ? 16u : 0u);
    }
  };
  load_step(0, 0);
  cp_async_commit();  // group: Q + step 0

  tc05::fence_before();
  __syncthreads();
  tc05::fence_after();
  const uint32_t tmem = *taddr_ptr;
  const uint32_t row_taddr = tmem + ((uint32_t)(32 * warp) << 16);
  const int row = tid;  // TMEM lane = query row
  const bool warp_busy = 32 * warp < nq;

  constexpr uint32_t fmt = std::is_same<T, __nv_bfloat16>::value ? 1u : 0u;
  constexpr uint32_t idesc_s = tc05::instr_desc_f16(fmt, S::kRows, S::kStep, 0, 0);
  constexpr uint32_t idesc_o = tc05::instr_desc_f16(fmt, S::kRows, D, 0, 1);

  float m_use = -INFINITY;  // reference max of O and l (base-2 scores)
  float l = 0.f;
  int err = 0;
  for (int i = 0; i < S::kSteps; ++i) {
    const int stage = i & 1;
    if (i > 0) {
      // MMA2 of step i-1 is done: O is current, P and the other stage are free.
      if (!tc05::mbar_wait_bounded(bar_o, (i - 1) & 1, kWaitCycles)) err = 1;
      tc05::fence_after();
    }
    if (i + 1 < S::kSteps && !err) load_step(i + 1, (i + 1) & 1);
    cp_async_commit();
    cp_async_wait<1>();
    tc05::fence_proxy_async_smem();
    tc05::fence_before();
    err = __syncthreads_or(err);
    if (err) break;
    const uint32_t kst = st_smem + stage * S::kStageBytes;
    const uint32_t vst = kst + S::kTileBytes;
    if (tid == 0) {
      tc05::fence_after();
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint32_t blk = ks >> 2, koff = (ks & 3) * 32;
        const uint64_t adesc = tc05::smem_desc_sw128(q_smem + blk * S::kQBlockBytes + koff, 16, 1024);
        const uint64_t bdesc = tc05::smem_desc_sw128(kst + blk * S::kKVBlockBytes + koff, 16, 1024);
        tc05::mma_ss(tmem + S::kSCol, adesc, bdesc, idesc_s, ks > 0 ? 1u : 0u);
      }
      tc05::commit(bar_s);
    }
    if (!tc05::mbar_wait_bounded(bar_s, i & 1, kWaitCycles)) err = 1;
    tc05::fence_after();
    if (warp_busy && !err) {
      // Validity of the step's 64 tokens: one bit per 16 tokens (block_size >= 16).
      const int tok0 = tok_begin + i * S::kStep;
      uint32_t sreg[2][32];
      tc05::ld32(row_taddr + S::kSCol, sreg[0]);
      tc05::ld32(row_taddr + S::kSCol + 32, sreg[1]);
      tc05::wait_ld();
      float mx = -INFINITY;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int q4 = 0; q4 < 2; ++q4) {
          const int tk = tok0 + 32 * h + 16 * q4;
          const bool ok = (unsigned)__shfl_sync(kFull, lane_page, tk / bs - first_block) < (unsigned)a.num_blocks;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float v = ok ? __uint_as_float(sreg[h][16 * q4 + j]) * a.qk_scale_log2 : -INFINITY;
            sreg[h][16 * q4 + j] = __float_as_uint(v);
            mx = fmaxf(mx, v);
          }
        }
      }
      // Lazy rescaling: keep the reference max unless the new max exceeds it by 8.
      float alpha = 1.f;
      if (mx > m_use + 8.f) {
        alpha = m_use == -INFINITY ? 0.f : exp2f(m_use - mx);
        m_use = mx;
      }
      const float ref = m_use == -INFINITY ? 0.f : m_use;
      float lsum = 0.f;
      uint32_t pk[32];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float p0 = exp2f(__uint_as_float(sreg[h][2 * j]) - ref);
          const float p1 = exp2f(__uint_as_float(sreg[h][2 * j + 1]) - ref);
          lsum += p0 + p1;
          pk[16 * h + j] = pack2<T>(p0, p1);
        }
      }
      l = l * alpha + lsum;
      if (i > 0 && __any_sync(kFull, alpha != 1.f)) {
#pragma unroll
        for (int cb = 0; cb < D / 32; ++cb) {
          uint32_t ov[32];
          tc05::ld32(row_taddr + S::kOCol + 32 * cb, ov);
          tc05::wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) ov[j] = __float_as_uint(__uint_as_float(ov[j]) * alpha);
          tc05::st32(row_taddr + S::kOCol + 32 * cb, ov);
        }
      }
      tc05::st32(row_taddr + S::kPCol, pk);
      tc05::wait_st();
    }
    tc05::fence_before();
    err = __syncthreads_or(err);
    if (err) break;
    if (tid == 0) {
      tc05::fence_after();
#pragma unroll
      for (int kt = 0; kt < S::kStep / 16; ++kt) {
        const uint64_t bdesc = tc05::smem_desc_sw128(vst + kt * 16 * 128, S::kKVBlockBytes, 1024);
        tc05::mma_ts(tmem + S::kOCol, tmem + S::kPCol + 8 * kt, bdesc, idesc_o, (i > 0 || kt > 0) ? 1u : 0u);
      }
      tc05::commit(bar_o);
    }
  }
  if (!err && !tc05::mbar_wait_bounded(bar_o, (S::kSteps - 1) & 1, kWaitCycles)) err = 1;
  err = __syncthreads_or(err);
  tc05::fence_after();
  if (!err && warp_busy) {
    const int64_t qrow = query_row(row);
    uint32_t ov[32];
    const float inv = l > 0.f ? 1.f / l : 0.f;
    const int64_t part = qrow * a.max_partitions + p;
#pragma unroll
    for (int cb = 0; cb < D / 32; ++cb) {
      tc05::ld32(row_taddr + S::kOCol + 32 * cb, ov);
      tc05::wait_ld();
      if (qrow >= 0) {
        float4* dst = reinterpret_cast<float4*>(a.o_part + part * D + 32 * cb);
#pragma unroll
        for (int j = 0; j < 8; ++j)
          dst[j] = make_float4(__uint_as_float(ov[4 * j]) * inv, __uint_as_float(ov[4 * j + 1]) * inv,
                               __uint_as_float(ov[4 * j + 2]) * inv, __uint_as_float(ov[4 * j + 3]) * inv);
      }
    }
    if (qrow >= 0) {
      a.m_part[part] = m_use == -INFINITY ? -INFINITY : m_use * kLn2;
      a.l_part[part] = l;
    }
  }
  if (err && tid == 0) flag_status(a.status, PA_DEV_TIMEOUT);
  cp_async_wait<0>();
  tc05::fence_before();
  __syncthreads();
  if (warp == 0) {
    tc05::fence_after();
    tc05::dealloc(tmem, S::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Warp-specialised, persistent shared-prefix kernel on tcgen05 (the default
// joint kernel).  One CTA per SM walks work items (chunk, kv head, shared
// partition) with stride gridDim.x; an item is 8 steps of 64 tokens.  Roles
// (8 warps):
//   warps 0-3  softmax: thread r owns query row r; per step it reads its S row
//              from TMEM, keeps the running max / sum (lazy rescaling of O),
//              writes P (16-bit) to TMEM; at the end of an item it writes the
//              partials.
//   warps 4-6  producers: K/V pages by TMA into a ring of STAGES buffers, as
//              far ahead as the ring allows, each warp a third of a step's
//              16-row boxes (one warp alone cannot issue boxes fast enough to
//              keep up with HBM); three steps before an item ends they start
//              the next item's queries (cp.async, one row per lane) into the
//              other query buffer, so the ring keeps filling across items.
//              Only they read the plan: each item's descriptor, table slice
//              and workspace rows reach the other roles through shared memory
//              with the queries (q_full); a descriptor marked invalid ends the
//              walk.
//   warp 7     MMA issuer (one lane): S(g) = Q.K^T into S[g & 1], then
//              O += P(g-1).V(g-1), so the tensor cores work on step g while
//              the softmax warps finish step g-1; an item's last O += P.V is
//              issued before the next item starts.
// Hand-offs are mbarriers, one per buffer, each waited at most one phase
// behind its next completion: s_full / s_free (S), p_full (P), o_done (MMA2,
// frees P, makes O current), kv_full / kv_empty (ring), q_full (queries and
// table slice), item_free (O and Q of an item read out).  Every wait is
// bounded; a timeout raises an abort flag that every role polls, then the CTA
// flags PA_DEV_TIMEOUT, lets its TMA loads land and its MMAs finish, frees
// TMEM and returns.
// ---------------------------------------------------------------------------
template <int D, int STAGES>
struct Tc05pShape {
  // TMA issue from one warp tops out near 41 GB/s per SM; three keep up with the step chain, and 8
  // warps in all (two per scheduler) leave each thread up to 255 registers.
  static constexpr int kProducerWarps = 3;
  // Warp w runs on scheduler w % 4.  The MMA warp takes scheduler 3: softmax
  // warp 0 (scheduler 0) has rows in every item, warp 3 only in full ones.
  static constexpr int kMmaWarp = 7;
  static constexpr int kThreads = 32 * (4 + kProducerWarps + 1);
  static_assert(kMmaWarp == 4 + kProducerWarps, "producers are warps 4 .. kMmaWarp - 1");
  static constexpr int kRows = 128;
  static constexpr int kStep = 64;
  static constexpr int kStepsPerItem = kPartition / kStep;  // 8
  static constexpr int kBlocks = D / 64;
  static constexpr int kQBlockBytes = kRows * 128;
  static constexpr int kQBytes = kBlocks * kQBlockBytes;
  static constexpr int kKVBlockBytes = kStep * 128;
  static constexpr int kTileBytes = kBlocks * kKVBlockBytes;
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kBoxBytes = 16 * 128;                 // one TMA box: 16 rows x 64 elements
  static constexpr int kBoxesPerStep = 2 * (kStep / 16) * kBlocks;
  static constexpr int kQOff = 0;
  static constexpr int kStageOff = 2 * kQBytes;
  static constexpr int kSliceOff = kStageOff + STAGES * kStageBytes;  // int32 [2][32] table slices
  static constexpr int kDescOff = kSliceOff + 256;                     // int32 [2][4] item descriptors
  static constexpr int kRowOff = kDescOff + 64;                        // int32 [2][kRows] workspace rows
  static constexpr int kBarOff = kRowOff + 2 * kRows * 4;
  // s_full, s_free, p_full, o_done, q_full, item_free x2; kv_full, kv_empty x STAGES; mma_drain
  static constexpr int kNumBars = 2 * 6 + 2 * STAGES + 1;
  static constexpr int kTaddrOff = kBarOff + 8 * kNumBars;
  static constexpr int kSmemBytes = kTaddrOff + 16 + 1024;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kSCol = 0, kPCol = 128, kOCol = 256;  // S[b] at 64b, P[b] at 128 + 32b, O[b] at 256 + 128b
  static_assert(D <= 128, "O double buffer needs D <= 128");
  // Producer pw issues boxes pw, pw + 3, ... and loads query rows pw * 32 + lane (+ 96).
  __host__ __device__ static constexpr int boxes_of(int pw) { return (kBoxesPerStep - pw + kProducerWarps - 1) / kProducerWarps; }
  static_assert(kBoxesPerStep <= 32 * kProducerWarps, "one lane per box");
  static_assert(kRows <= 64 * kProducerWarps && kRows > 32 * kProducerWarps, "one or two query rows per lane");
  static_assert(kQBytes >= 4 * 32 * 20 * 4, "the epilogue's four 32-row float tiles fit in a query buffer");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

struct SharedItem {
  int c, kvh, p, leader, moff, mcount;
  bool valid;
};

// Whether a plan entry names a work item whose arrays are all in range.
__device__ __forceinline__ bool shared_item_ok(const SharedItem& it, const DecodeArgs& a, int num_members,
                                               int num_seqs) {
  return (unsigned)it.leader < (unsigned)num_seqs && it.moff >= 0 && it.mcount >= 0 &&
         (int64_t)it.moff + it.mcount <= num_members && (int64_t)it.mcount * a.group <= 128 &&
         (int64_t)(it.p + 1) * kPartition <= (int64_t)a.max_blocks_per_seq * a.block_size &&
         it.p < a.max_partitions;
}

// The next usable work item at or after `cursor` (stride gridDim.x), in the
// order (partition, kv head, chunk) so concurrent CTAs share pages through L2.
// Entries that would index outside an array are reported and skipped.
__device__ __forceinline__ SharedItem next_shared_item(int64_t& cursor, int64_t total, int num_chunks,
                                                       const DecodeArgs& a, const int32_t* __restrict__ chunks,
                                                       int num_members, int num_seqs, bool report) {
  SharedItem it{};
  it.valid = false;
  while (cursor < total) {
    const int64_t w = cursor;
    cursor += gridDim.x;
    const int c = (int)(w % num_chunks);
    const int64_t rest = w / num_chunks;
    it.c = c;
    it.kvh = (int)(rest % a.num_kv_heads);
    it.p = (int)(rest / a.num_kv_heads);
    if (it.p >= __ldg(chunks + 4 * c + 3)) continue;
    it.leader = __ldg(chunks + 4 * c);
    it.moff = __ldg(chunks + 4 * c + 1);
    it.mcount = __ldg(chunks + 4 * c + 2);
    if (!shared_item_ok(it, a, num_members, num_seqs)) {
      if (report) flag_status(a.status, PA_DEV_BAD_PLAN);
      continue;
    }
    it.valid = true;
    return it;
  }
  return it;
}

// The same walk split in two, so that the plan loads of the next item overlap
// the current one: `prefetch_shared_item` takes the next work index and starts
// loading its chunk's entries; `resolve_shared_item` uses them once they are
// needed, continuing the walk where the index is not a usable item.
struct SharedItemPrefetch {
  int64_t w;  // work index, -1 past the end
  int sp, leader, moff, mcount;
};

__device__ __forceinline__ SharedItemPrefetch prefetch_shared_item(int64_t& cursor, int64_t total, int num_chunks,
                                                                   const int32_t* __restrict__ chunks) {
  SharedItemPrefetch f{-1, 0, 0, 0, 0};
  if (cursor < total) {
    f.w = cursor;
    cursor += gridDim.x;
    const int c = (int)(f.w % num_chunks);
    f.sp = __ldg(chunks + 4 * c + 3);
    f.leader = __ldg(chunks + 4 * c);
    f.moff = __ldg(chunks + 4 * c + 1);
    f.mcount = __ldg(chunks + 4 * c + 2);
  }
  return f;
}

__device__ __forceinline__ SharedItem resolve_shared_item(const SharedItemPrefetch& f, int64_t& cursor, int64_t total,
                                                          int num_chunks, const DecodeArgs& a,
                                                          const int32_t* __restrict__ chunks, int num_members,
                                                          int num_seqs, bool report) {
  SharedItem it{};
  it.valid = false;
  if (f.w < 0) return it;
  const int64_t rest = f.w / num_chunks;
  it.c = (int)(f.w % num_chunks);
  it.kvh = (int)(rest % a.num_kv_heads);
  it.p = (int)(rest / a.num_kv_heads);
  if (it.p < f.sp) {
    it.leader = f.leader;
    it.moff = f.moff;
    it.mcount = f.mcount;
    if (shared_item_ok(it, a, num_members, num_seqs)) {
      it.valid = true;
      return it;
    }
    if (report) flag_status(a.status, PA_DEV_BAD_PLAN);
  }
  return next_shared_item(cursor, total, num_chunks, a, chunks, num_members, num_seqs, report);
}

template <typename T, int D, int STAGES>
__global__ void __launch_bounds__(Tc05pShape<D, STAGES>::kThreads, 1)
    decode_shared_tc05p_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tmap_k,
                               const __grid_constant__ CUtensorMap tmap_v, const int32_t* __restrict__ chunks,
                               int num_chunks, const int32_t* __restrict__ members, int num_members, int num_seqs,
                               int max_shared_partitions, int fault) {
  using S = Tc05pShape<D, STAGES>;
  constexpr int SPI = S::kStepsPerItem;
  static_assert(SPI >= 3, "the next item's queries are loaded three steps before the item ends");
  extern __shared__ uint8_t smem_raw[];
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int bs = a.block_size;
  const int G = a.group;
  const int64_t total_rows = (int64_t)a.num_blocks * a.num_kv_heads * bs;
  const int64_t total_items = (int64_t)max_shared_partitions * a.num_kv_heads * num_chunks;

  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw);
  int32_t* tslice = reinterpret_cast<int32_t*>(base_ptr + S::kSliceOff);  // [2][32]
  // Written by the producers, published with q_full: the item in buffer b
  // (valid, partition, kv head, member count; valid 0 ends the walk) and the
  // workspace row of each of its query rows (-1: none).
  volatile int32_t* desc = reinterpret_cast<volatile int32_t*>(base_ptr + S::kDescOff);  // [2][4]
  int32_t* prow_s = reinterpret_cast<int32_t*>(base_ptr + S::kRowOff);                   // [2][kRows]
  const uint32_t bar0 = base + S::kBarOff;
  auto s_full = [&](int b) { return bar0 + 8u * b; };
  auto s_free = [&](int b) { return bar0 + 16u + 8u * b; };
  auto p_full = [&](int b) { return bar0 + 32u + 8u * b; };
  auto o_done = [&](int b) { return bar0 + 48u + 8u * b; };
  auto q_full = [&](int b) { return bar0 + 64u + 8u * b; };
  auto item_free = [&](int b) { return bar0 + 80u + 8u * b; };
  auto kv_full = [&](int st) { return bar0 + 96u + 8u * st; };
  auto kv_empty = [&](int st) { return bar0 + 96u + 8u * STAGES + 8u * st; };
  const uint32_t mma_drain = bar0 + 96u + 16u * STAGES;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base_ptr + S::kTaddrOff + 8);
  const uint32_t taddr_slot = base + S::kTaddrOff;

  // Bounded wait that also gives up once another role has aborted.  A waiting
  // thread sleeps until the phase completes (woken by the completion, or
  // after 20 us to look at the abort flag), so waiting warps leave the issue
  // slots to the softmax warps they share a scheduler with.
  auto wait = [&](uint32_t bar, uint32_t parity) -> bool {
    const long long t0 = clock64();
    while (!tc05::mbar_try_wait_sleep(bar, parity, 20000u)) {
      if (*abort_flag) return false;
      if (clock64() - t0 > kWaitCycles) {
        *abort_flag = 1;
        return false;
      }
    }
    return true;
  };

  // Warp-uniform form of `wait` for the softmax and producer warps: every lane
  // waits (bounded) and the warp agrees on the outcome, so a break is taken by
  // all 32 lanes together and no lane is left behind at a __syncwarp.
  auto wwait = [&](uint32_t bar, uint32_t parity) -> bool { return __all_sync(kFull, wait(bar, parity)); };

  // -- set-up -----------------------------------------------------------------------------------
  if (tid == 0) {
    for (int b = 0; b < 2; ++b) {
      tc05::mbar_init(s_full(b), 1);
      tc05::mbar_init(s_free(b), 4);     // one arrival per softmax warp
      tc05::mbar_init(p_full(b), 4);
      tc05::mbar_init(o_done(b), 1);
      tc05::mbar_init(q_full(b), S::kProducerWarps);  // lane 0 of each producer warp
      tc05::mbar_init(item_free(b), 4);
    }
    for (int st = 0; st < STAGES; ++st) {
      tc05::mbar_init(kv_full(st), S::kProducerWarps);
      tc05::mbar_init(kv_empty(st), 1);
    }
    tc05::mbar_init(mma_drain, 1);
    *abort_flag = 0;
    tc05::fence_mbar_init();
    tc05::prefetch_tensormap(&tmap_k);
    tc05::prefetch_tensormap(&tmap_v);
  }
  if (warp == 0) {
    tc05::alloc(taddr_slot, S::kTmemCols);
    tc05::relinquish();
  }
  tc05::fence_before();
  __syncthreads();
  tc05::fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(base_ptr + S::kTaddrOff);

  // The per-sequence partition kernel that follows may start on SMs this grid
  // leaves (its CTAs cannot share an SM with this one's).
  if (tid == 0) asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  int64_t cursor = blockIdx.x;
  int64_t prod_g = 0;  // producer: steps whose loads have been issued
  if (warp >= 4 && warp != S::kMmaWarp) {
    // ---------------------------------------------------------------- producers
    const int pw = warp < S::kMmaWarp ? warp - 4 : warp - 5;
    const T* qbase = reinterpret_cast<const T*>(a.q);
    // Table entries of `it` (lane l holds page l of the partition; -1 past its end).
    auto load_pages = [&](const SharedItem& it) -> int {
      const int fb = it.p * kPartition / bs;
      const int nblk = (it.p * kPartition + kPartition - 1) / bs - fb + 1;
      return lane < nblk ? __ldg(a.block_tables + (int64_t)it.leader * a.max_blocks_per_seq + fb + lane) : -1;
    };
    // Query rows pw * 32 + lane (+ 96) of `it` (zero past mcount * G) into buffer qb;
    // the first producer warp also stores the table slice for the softmax warps.
    auto load_q = [&](const SharedItem& it, int qb, int pages) {
      const uint32_t qs = base + S::kQOff + qb * S::kQBytes;
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int r = pw * 32 + lane + 32 * S::kProducerWarps * k;
        if (r >= S::kRows) break;
        int64_t row = -1;
        if (r < it.mcount * G) {
          const int mi = r / G;
          const int b = __ldg(members + it.moff + mi);
          if ((unsigned)b < (unsigned)num_seqs) row = (int64_t)b * a.num_q_heads + it.kvh * G + (r - mi * G);
        }
        const T* src = qbase + (row < 0 ? 0 : row) * D;
#pragma unroll
        for (int ck = 0; ck < D / 8; ++ck)
          cp_async_16(qs + (ck >> 3) * S::kQBlockBytes + r * 128 + (((ck & 7) ^ (r & 7)) << 4), src + ck * 8,
                      row < 0 ? 0u : 16u);
        prow_s[qb * S::kRows + r] = row < 0 ? -1 : (int32_t)(row * a.max_partitions + it.p);
      }
      if (pw == 0) {
        tslice[qb * 32 + lane] = pages;
        if (lane == 0) {
          desc[qb * 4 + 1] = it.p;
          desc[qb * 4 + 2] = it.kvh;
          desc[qb * 4 + 3] = it.mcount;
          desc[qb * 4 + 0] = 1;
        }
      }
      cp_async_commit();
    };
    auto end_walk = [&](int qb) {  // buffer qb holds no item: the other roles stop there
      if (pw == 0 && lane == 0) desc[qb * 4 + 0] = 0;
    };
    auto publish_q = [&](int qb) {  // after load_q: make it visible, then signal
      cp_async_wait<0>();
      tc05::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(q_full(qb)) : "memory");
    };
    SharedItem it = next_shared_item(cursor, total_items, num_chunks, a, chunks, num_members, num_seqs,
                                     pw == 0 && lane == 0);
    int my_page = -1;
    if (it.valid) {
      my_page = load_pages(it);
      load_q(it, 0, my_page);
    } else {
      end_walk(0);
    }
    if (fault != PA_FAULT_WITHHOLD_FIRST_ITEM) publish_q(0);
    else cp_async_wait<0>();  // test hook: the other roles' waits for this hand-off run out
    int64_t g = 0;
    for (int j = 0; it.valid; ++j) {
      const int qb = j & 1;
      const SharedItemPrefetch pf = prefetch_shared_item(cursor, total_items, num_chunks, chunks);
      SharedItem nxt{};
      nxt.valid = false;
      const int fb = it.p * kPartition / bs;
      int nxt_page = -1;
      bool stop = false;
      for (int i = 0; i < SPI; ++i, ++g) {
        const int st = (int)(g % STAGES);
        if (g >= STAGES && !wwait(kv_empty(st), (uint32_t)(((g - STAGES) / STAGES) & 1))) { stop = true; break; }
        if (lane == 0) tc05::mbar_arrive_expect_tx(kv_full(st), S::boxes_of(pw) * S::kBoxBytes);
        // box -> (row box rb, 64-wide block blk, K or V)
        const int box = pw + S::kProducerWarps * lane;
        const int kv = box & 1;
        const int blk = (box >> 1) % S::kBlocks;
        const int rb = ((box >> 1) / S::kBlocks) % (S::kStep / 16);
        const int tok = it.p * kPartition + i * S::kStep + 16 * rb;
        const int page = __shfl_sync(kFull, my_page, tok / bs - fb);
        __syncwarp();
        if (box < S::kBoxesPerStep) {
          const int64_t y = (unsigned)page < (unsigned)a.num_blocks
                                ? ((int64_t)page * a.num_kv_heads + it.kvh) * bs + tok % bs
                                : total_rows;  // out of range: the box is filled with zeros
          const uint32_t dst = base + S::kStageOff + st * S::kStageBytes + kv * S::kTileBytes +
                               blk * S::kKVBlockBytes + rb * S::kBoxBytes;
          tc05::tma_load_2d(dst, kv ? (const void*)&tmap_v : (const void*)&tmap_k, kv_full(st), 64 * blk, (int32_t)y);
        }
        __syncwarp();
        if (pw == 0) prod_g = g + 1;
        // Three steps before the end: the next item's queries go into the other
        // buffer once the item that last used it (j - 1) has been read out.
        if (i == SPI - 3) {
          nxt = resolve_shared_item(pf, cursor, total_items, num_chunks, a, chunks, num_members, num_seqs,
                                    pw == 0 && lane == 0);
          if (j >= 1 && !wwait(item_free(qb ^ 1), (uint32_t)(((j - 1) >> 1) & 1))) { stop = true; break; }
          if (nxt.valid) {
            nxt_page = load_pages(nxt);
            load_q(nxt, qb ^ 1, nxt_page);
          } else {
            end_walk(qb ^ 1);
          }
        }
      }
      if (stop || __any_sync(kFull, *abort_flag != 0)) break;
      publish_q(qb ^ 1);
      it = nxt;
      my_page = nxt_page;
    }
    cp_async_wait<0>();  // nothing may land in shared memory after the CTA leaves
  } else if (warp == S::kMmaWarp) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t fmt = std::is_same<T, __nv_bfloat16>::value ? 1u : 0u;
      constexpr uint32_t idesc_s = tc05::instr_desc_f16(fmt, S::kRows, S::kStep, 0, 0);
      constexpr uint32_t idesc_o = tc05::instr_desc_f16(fmt, S::kRows, D, 0, 1);
      auto mma2 = [&](int64_t gp) -> bool {  // O[item of gp] += P(gp) . V(gp)
        if (!wait(p_full((int)(gp & 1)), (uint32_t)((gp >> 1) & 1))) return false;
        tc05::fence_after();
        const int st = (int)(gp % STAGES);
        const uint32_t vs = base + S::kStageOff + st * S::kStageBytes + S::kTileBytes;
        const uint32_t ocol = S::kOCol + 128u * (uint32_t)((gp / SPI) & 1);
        const int ip = (int)(gp % SPI);
#pragma unroll
        for (int kt = 0; kt < S::kStep / 16; ++kt)
          tc05::mma_ts(tmem + ocol, tmem + S::kPCol + 32 * (uint32_t)(gp & 1) + 8 * kt,
                       tc05::smem_desc_sw128(vs + kt * 16 * 128, S::kKVBlockBytes, 1024), idesc_o,
                       (ip > 0 || kt > 0) ? 1u : 0u);
        tc05::commit(o_done((int)(gp & 1)));
        tc05::commit(kv_empty(st));
        return true;
      };
      int64_t g = 0;
      bool ok = true;
      for (int j = 0; ok; ++j) {
        const int qb = j & 1;
        if (!wait(q_full(qb), (uint32_t)((j >> 1) & 1))) break;
        if (desc[qb * 4 + 0] == 0) break;  // the walk has ended
        tc05::fence_after();
        tc05::fence_proxy_async_smem();
        const uint32_t qs = base + S::kQOff + qb * S::kQBytes;
        for (int i = 0; i < SPI; ++i, ++g) {
          const int st = (int)(g % STAGES);
          if (!wait(kv_full(st), (uint32_t)((g / STAGES) & 1))) { ok = false; break; }
          if (g >= 2 && !wait(s_free((int)(g & 1)), (uint32_t)(((g - 2) >> 1) & 1))) { ok = false; break; }
          tc05::fence_after();
          const uint32_t ks = base + S::kStageOff + st * S::kStageBytes;
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t blk = k >> 2, koff = (k & 3) * 32;
            tc05::mma_ss(tmem + S::kSCol + 64 * (uint32_t)(g & 1),
                         tc05::smem_desc_sw128(qs + blk * S::kQBlockBytes + koff, 16, 1024),
                         tc05::smem_desc_sw128(ks + blk * S::kKVBlockBytes + koff, 16, 1024), idesc_s,
                         k > 0 ? 1u : 0u);
          }
          tc05::commit(s_full((int)(g & 1)));
          if (i >= 1 && !mma2(g - 1)) { ok = false; break; }
        }
        // Close the item (its epilogue must not wait for the next item's queries).
        if (ok && !mma2(g - 1)) ok = false;
      }
      // Every MMA this thread issued has completed before the CTA frees TMEM and
      // shared memory (on an abort some may still be running).
      tc05::commit(mma_drain);
      {
        const long long t0 = clock64();
        while (!tc05::mbar_try_wait(mma_drain, 0) && clock64() - t0 < kWaitCycles) {
        }
      }
    }
  } else {
    // ---------------------------------------------------------------- softmax warps 0-3
    const uint32_t row_t = tmem + ((uint32_t)(32 * warp) << 16);
    int64_t g = 0;
    for (int j = 0;; ++j) {
      const int qb = j & 1;
      if (!wwait(q_full(qb), (uint32_t)((j >> 1) & 1))) break;  // item, table slice and rows
      if (desc[qb * 4 + 0] == 0) break;                          // the walk has ended
      SharedItem it{};
      it.p = desc[qb * 4 + 1];
      it.mcount = desc[qb * 4 + 3];
      const bool busy = 32 * warp < it.mcount * G;
      // Page validity of the item's 32 16-token groups (4 per step), one lane each.
      static_assert(kPartition / 16 == 32 && S::kStep == 64, "one lane per 16-token group of an item");
      const uint32_t page_ok = __ballot_sync(
          kFull, (unsigned)tslice[qb * 32 + (it.p * kPartition + 16 * lane) / bs - it.p * kPartition / bs] <
                     (unsigned)a.num_blocks);
      float m_use = -INFINITY, l = 0.f;
      bool ok = true;
      for (int i = 0; i < SPI; ++i, ++g) {
        if (!wwait(s_full((int)(g & 1)), (uint32_t)((g >> 1) & 1))) { ok = false; break; }
        tc05::fence_after();
        uint32_t sreg[2][32];
        if (busy) {
          tc05::ld32(row_t + S::kSCol + 64 * (uint32_t)(g & 1), sreg[0]);
          tc05::ld32(row_t + S::kSCol + 64 * (uint32_t)(g & 1) + 32, sreg[1]);
          tc05::wait_ld();
        }
        tc05::fence_before();
        __syncwarp();
        if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(s_free((int)(g & 1))) : "memory");
        uint32_t pk[32];
        float alpha = 1.f;
        if (busy) {
          const int bad = (int)(~page_ok >> (4 * i)) & 0xF;  // 16-token groups whose page is out of range
          float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
          float nref;  // minus the reference score; weights are 2^(s * scale + nref)
          if (bad == 0 && a.qk_scale_log2 > 0.f) {
            // Every score is finite: max over the raw scores, one FMA per weight.
#pragma unroll
            for (int e = 0; e < 64; ++e) mx4[e & 3] = fmaxf(mx4[e & 3], __uint_as_float(sreg[e >> 5][e & 31]));
            const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * a.qk_scale_log2;
            if (mx > m_use + 8.f) {
              alpha = m_use == -INFINITY ? 0.f : ex2_approx(m_use - mx);
              m_use = mx;
            }
            nref = -m_use;
            float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int jj = 0; jj < 32; ++jj) {
              const int e0 = 2 * jj, e1 = 2 * jj + 1;
              const float p0 = ex2_approx(fmaf(__uint_as_float(sreg[e0 >> 5][e0 & 31]), a.qk_scale_log2, nref));
              const float p1 = ex2_approx(fmaf(__uint_as_float(sreg[e1 >> 5][e1 & 31]), a.qk_scale_log2, nref));
              ls[jj & 3] += p0 + p1;
              pk[jj] = pack2<T>(p0, p1);
            }
            l = l * alpha + ((ls[0] + ls[1]) + (ls[2] + ls[3]));
          } else {
            // Scores of tokens on an out-of-range page are -inf (weight 0).
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
#pragma unroll
              for (int jj = 0; jj < 16; ++jj) {
                const int e = 16 * q4 + jj;
                const float v = (bad >> q4) & 1 ? -INFINITY : __uint_as_float(sreg[e >> 5][e & 31]) * a.qk_scale_log2;
                sreg[e >> 5][e & 31] = __float_as_uint(v);
                mx4[jj & 3] = fmaxf(mx4[jj & 3], v);
              }
            }
            const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
            if (mx > m_use + 8.f) {
              alpha = m_use == -INFINITY ? 0.f : ex2_approx(m_use - mx);
              m_use = mx;
            }
            nref = m_use == -INFINITY ? 0.f : -m_use;
            float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int jj = 0; jj < 32; ++jj) {
              const int e0 = 2 * jj, e1 = 2 * jj + 1;
              const float p0 = ex2_approx(__uint_as_float(sreg[e0 >> 5][e0 & 31]) + nref);
              const float p1 = ex2_approx(__uint_as_float(sreg[e1 >> 5][e1 & 31]) + nref);
              ls[jj & 3] += p0 + p1;
              pk[jj] = pack2<T>(p0, p1);
            }
            l = l * alpha + ((ls[0] + ls[1]) + (ls[2] + ls[3]));
          }
        }
        if (busy && i > 0 && __any_sync(kFull, alpha != 1.f)) {
          // O is current once O += P.V of step g - 1 has completed.
          if (!wwait(o_done((int)((g - 1) & 1)), (uint32_t)(((g - 1) >> 1) & 1))) { ok = false; break; }
          tc05::fence_after();
          const uint32_t ocol = S::kOCol + 128u * (uint32_t)qb;
#pragma unroll 1
          for (int cb = 0; cb < D / 16; ++cb) {
            uint32_t ov[16];
            tc05::ld16(row_t + ocol + 16 * cb, ov);
            tc05::wait_ld();
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) ov[jj] = __float_as_uint(__uint_as_float(ov[jj]) * alpha);
            tc05::st16(row_t + ocol + 16 * cb, ov);
          }
        }
        // P buffer g & 1 was last read by O += P.V of step g - 2.
        if (g >= 2 && !wwait(o_done((int)(g & 1)), (uint32_t)(((g - 2) >> 1) & 1))) { ok = false; break; }
        tc05::fence_after();
        if (busy) {
          tc05::st32(row_t + S::kPCol + 32 * (uint32_t)(g & 1), pk);
          tc05::wait_st();
        }
        tc05::fence_before();
        __syncwarp();
        if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(p_full((int)(g & 1))) : "memory");
      }
      if (!ok) break;
      // Epilogue: the item's last O += P.V (step g - 1) has to complete.
      const int64_t gl = g - 1;
      if (!wwait(o_done((int)(gl & 1)), (uint32_t)((gl >> 1) & 1))) break;
      tc05::fence_after();
      if (busy) {
        const int32_t prow = prow_s[qb * S::kRows + tid];  // workspace row of this thread's partial
        const float inv = l > 0.f ? 1.f / l : 0.f;
        const uint32_t ocol = S::kOCol + 128u * (uint32_t)qb;
        // O leaves through a 32-row tile per warp (rows 80 bytes apart: 16-byte
        // accesses are conflict-free both ways) in this item's query buffer,
        // idle once the item's MMAs are done and not refilled before item_free,
        // 16 columns at a time.  Store instructions cost the most here, so each
        // one writes 16 bytes per lane: 64 contiguous bytes of each of 8 rows.
        constexpr int kTileStride = 20;  // floats
        float* tile = reinterpret_cast<float*>(base_ptr + S::kQOff + qb * S::kQBytes) + warp * 32 * kTileStride;
        float4* wr = reinterpret_cast<float4*>(tile + lane * kTileStride);  // this thread's row
        const int rsub = lane >> 2, csub = lane & 3;                        // row 8i + rsub, 4 columns
#pragma unroll 1
        for (int cb = 0; cb < D / 16; ++cb) {
          uint32_t ov[16];
          tc05::ld16(row_t + ocol + 16 * cb, ov);
          tc05::wait_ld();
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4)
            wr[q4] = make_float4(__uint_as_float(ov[4 * q4]) * inv, __uint_as_float(ov[4 * q4 + 1]) * inv,
                                 __uint_as_float(ov[4 * q4 + 2]) * inv, __uint_as_float(ov[4 * q4 + 3]) * inv);
          __syncwarp();
          float4 v[4];
          int32_t pr[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            pr[i] = __shfl_sync(kFull, prow, 8 * i + rsub);
            v[i] = *reinterpret_cast<const float4*>(tile + (8 * i + rsub) * kTileStride + 4 * csub);
          }
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 4; ++i)
            if (pr[i] >= 0) *reinterpret_cast<float4*>(a.o_part + (int64_t)pr[i] * D + 16 * cb + 4 * csub) = v[i];
        }
        if (prow >= 0) {
          a.m_part[prow] = m_use == -INFINITY ? -INFINITY : m_use * kLn2;
          a.l_part[prow] = l;
        }
      }
      tc05::fence_before();
      __syncwarp();
      if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(item_free(qb)) : "memory");
    }
  }

  // -- teardown ---------------------------------------------------------------------------------
  __syncthreads();
  if (*abort_flag) {
    if (tid == 0) flag_status(a.status, PA_DEV_TIMEOUT);
    // Let the TMA loads still in the ring land before the shared memory is released
    // (the last STAGES issued steps; each stage's latest phase is at most one behind).
    if (warp == 4 && lane == 0)  // (a phase another producer warp left short runs into the bound)
      for (int64_t gl = prod_g > STAGES ? prod_g - STAGES : 0; gl < prod_g; ++gl) {
        const long long t0 = clock64();
        while (!tc05::mbar_try_wait(kv_full((int)(gl % STAGES)), (uint32_t)((gl / STAGES) & 1)) &&
               clock64() - t0 < kWaitCycles) {
        }
      }
  }
  cp_async_wait<0>();
  tc05::fence_before();
  __syncthreads();
  if (warp == 0) {
    tc05::fence_after();
    tc05::dealloc(tmem, S::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Balanced shared-prefix kernel on tcgen05 (the default joint kernel).  One
// persistent CTA per SM covers a share of the whole call:
//   shared steps   the 64-token steps of every (kv head, chunk) lane that all of
//                  the chunk's members share (its whole shared partitions), and
//   tail steps     every (kv head, member) lane from the end of the member's
//                  shared partitions to its context length.
// Shared steps are split evenly over the CTAs in contiguous ranges (a range
// may end in one lane and go on in the next); a tail lane goes whole to the
// CTA whose range holds its start, weighed as its steps plus kEpilogueSteps
// for its epilogue, so that the CTAs finish together and no per-sequence
// kernel has to follow for the members.  A CTA's run of consecutive steps in
// one lane is a segment: for each of its query rows it writes one partial
// (o / l, m, l) into a workspace slot of the lane's partitions -- the k-th
// segment of a lane takes the lane's k-th slot -- and the segment that ends
// the lane writes l = 0 into the lane's slots left over, which the merge skips.
// A lane has no more segments than partitions: CTA ranges are at least 16
// steps long, and no range ends inside a lane of one partition.
//
// Roles (9 warps):
//   warps 0-3       softmax: thread r owns query row r (TMEM lane r), as in the
//                   per-partition kernel; a tail segment masks the tokens past
//                   its member's context, and every step masks the 16-token
//                   groups whose page is out of range (bits the producers
//                   publish with the stage).
//   warps 4-6, 8    producers: producer k loads 16-token group k of every step
//                   -- its page's K and V slabs, 16-byte cp.async copies into
//                   the 128-byte-swizzled stage, their completion tracked by the
//                   stage's mbarrier -- with the page numbers of 32 steps held
//                   one per lane (the next 32 already requested); three steps
//                   before a segment ends they load the next segment's query
//                   rows (one per lane), descriptor and workspace rows.
//   warp 7          MMA issuer (one lane): S(g) = Q.K^T, then O += P(g-1).V(g-1).
// Hand-offs, bounded waits, the abort path and the fault hook are those of
// the per-partition kernel.
// ---------------------------------------------------------------------------
template <int D, int STAGES>
struct SegShape {
  // Four producer warps, one 16-token group of every step each (measured: seven,
  // sharing every step's copies, were slower -- the softmax warps then share
  // their schedulers with two producers each).
  static constexpr int kProducerWarps = 4;
  static constexpr int kMmaWarp = 7;
  static constexpr int kThreads = 32 * 9;
  static constexpr int kRows = 128;
  static constexpr int kStep = 64;
  static constexpr int kBlocks = D / 64;
  static constexpr int kQBlockBytes = kRows * 128;
  static constexpr int kQBytes = kBlocks * kQBlockBytes;
  static constexpr int kKVBlockBytes = kStep * 128;
  static constexpr int kTileBytes = kBlocks * kKVBlockBytes;
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kChunksPerRow = D / 8;         // 16-byte chunks of one K or V row
  static constexpr int kRowsPerCopy = 32 / kChunksPerRow;  // rows one warp-wide copy covers
  static constexpr int kCopiesPerGroup = 16 / kRowsPerCopy;

  static constexpr int kQOff = 0;
  static constexpr int kStageOff = 2 * kQBytes;
  static constexpr int kDescOff = kStageOff + STAGES * kStageBytes;            // int32 [2][16]
  static constexpr int kRowOff = kDescOff + 128;                               // int32 [2][kRows]
  static constexpr int kBarOff = kRowOff + 2 * kRows * 4;
  // s_full, p_full, o_done, q_full, item_free x2; kv_full, kv_empty x STAGES; mma_drain
  static constexpr int kNumBars = 2 * 5 + 2 * STAGES + 1;
  static constexpr int kTaddrOff = kBarOff + 8 * kNumBars;
  static constexpr int kSmemBytes = kTaddrOff + 16 + 1024;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kSCol = 0, kPCol = 128, kOCol = 256;  // S[b] at 64b, P[b] at 128 + 32b, O[b] at 256 + 128b
  static constexpr int kEpilogueSteps = 2;  // weight of a tail lane's epilogue, in steps
  static_assert(D <= 128, "O double buffer needs D <= 128");
  static_assert(kRows == 32 * 4, "one query row per lane of the first four producer warps");
  static_assert(kStep == 16 * 4, "four 16-token groups per step");
  static_assert(kQBytes >= 4 * 32 * 20 * 4, "the epilogue's four 32-row float tiles fit in a query buffer");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
  // Producer warp index of warp w (warps 4-6 and 8).
  __host__ __device__ static constexpr int producer_of(int w) { return w < kMmaWarp ? w - 4 : w - 5; }
};

// Chunk c of a plan, its lane length in 64-token steps: a shared-prefix plan
// gives whole partitions (8 steps each), a verify plan (vt = T > 0) the steps
// that cover the leader's context.  An entry that would index outside an array
// is reported (when `report`) and read as an empty chunk.
struct SegChunk {
  int leader, moff, mcount, ns;
};
__device__ __forceinline__ SegChunk seg_chunk(const DecodeArgs& a, const int32_t* __restrict__ chunks, int c,
                                             int num_members, int num_seqs, bool report, int vt) {
  SegChunk k{__ldg(chunks + 4 * c), __ldg(chunks + 4 * c + 1), __ldg(chunks + 4 * c + 2), __ldg(chunks + 4 * c + 3)};
  const int64_t steps = vt > 0 ? (int64_t)k.ns : 8 * (int64_t)k.ns;
  const bool ok = (unsigned)k.leader < (unsigned)num_seqs && k.moff >= 0 && k.mcount >= 0 &&
                  (int64_t)k.moff + k.mcount <= num_members && (int64_t)k.mcount * a.group <= 128 && steps >= 0 &&
                  64 * (steps - 1) < (int64_t)a.max_blocks_per_seq * a.block_size &&
                  (steps + 7) / 8 <= a.max_partitions;
  if (!ok) {
    if (report) flag_status(a.status, PA_DEV_BAD_PLAN);
    k.mcount = 0;
  }
  k.ns = k.mcount == 0 ? 0 : (int)steps;
  return k;
}

// A segment: steps [s0, s1) of one lane.  kind 0 = shared (rows: the chunk's
// members), 1 = tail (rows: member `b`); `leader` is the sequence whose block
// table gives the pages; tokens at or past `ctx` are read as nothing.  Row r
// (member mi = r / G) sees the tokens before ctx - max(0, causal - mi): a verify
// chunk's tokens first .. first + count - 1 of T sit at the context's last T
// positions, so causal = T - 1 - first; 0 elsewhere.  Its partial goes to
// workspace slot `slot`; slots [slot + 1, mark_end) are marked empty.  A verify
// segment that covers its whole lane (`final`) writes its rows' outputs instead
// and marks slot 0 done (l = -1), so that the merge leaves those rows alone.
struct Seg {
  int kind, kvh, leader, moff, mcount, b, s0, s1, ctx, slot, mark_end, causal, final;
};

// The segments of one CTA, in order.  Every lane of a producer warp runs the
// same walk (warp-uniform results); every producer warp runs its own copy.
// All unit counts stay below kSegMaxUnits (the launcher checks an upper bound),
// so the walk runs in 32-bit arithmetic: total * k for k <= 148 CTAs fits.
constexpr int kSegMaxUnits = 1 << 23;
struct SegWalk {
  int u0, u1;          // this CTA's range of weighted units
  int total;           // units of the whole call
  int ctas;            // CTAs with a range
  int base;            // units of all shared lanes: H_kv * S_sh
  int s_sh, tw;        // shared steps per kv head; tail weight per kv head
  // shared lanes
  int su, su_end;      // next shared unit, end of this CTA's shared units
  int skvh, sc, soff;  // lane (kv head, chunk) of unit su and its offset in the lane
  SegChunk sci;
  SegChunk cl;         // plans of at most 32 chunks: chunk `lane` of this lane
  int cl_incl;         // and the lanes' units of chunks 0 .. lane
  // tail lanes: sequences [tm0, tm0 + 32) of kv head tkvh, weighted start tw_at
  int tkvh, tm0;
  int tw_at;
  uint32_t tmask;      // members of the loaded batch still to hand out
  bool tloaded, tdone;
  int tT, tfp, tctx;      // per lane: tail steps, first tail partition and context of sequence tm0 + lane
  int vt;                 // verify plans: query tokens per sequence (0: a shared-prefix plan)
};

// Tail of batch sequence b: its steps from the end of its shared partitions
// to its context (0 for a sequence outside every group), first tail partition
// and context.
__device__ __forceinline__ void seg_tail_of(const DecodeArgs& a, const int32_t* __restrict__ first_partition, int b,
                                            int num_seqs, int& T, int& fp, int& ctx) {
  T = 0;
  fp = 0;
  ctx = 0;
  if (b < num_seqs) {
    fp = __ldg(first_partition + b);
    ctx = context_of(a, b, false);
    if (fp <= 0 || fp > a.max_partitions) fp = 0;
    else T = max(0, (ctx + 63) / 64 - 8 * fp);
  }
}

// Warp-wide inclusive sum.
__device__ __forceinline__ int warp_incl_sum(int v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(kFull, v, off);
    if (lane >= off) v += o;
  }
  return v;
}

// Units of shared lane (kv head, c): kSegLeadIn units that carry no step (the
// cost of starting a segment: the previous one's epilogue and the switch of
// query rows), then one unit per 64-token step of the lane.
constexpr int kSegLeadIn = 3;
__device__ __forceinline__ int seg_lane_units(int ns) { return ns > 0 ? ns + kSegLeadIn : 0; }

// Chunk c of the plan from the lane registers of the walk (plans of at most 32
// chunks: lane c holds chunk c) or from global memory.
__device__ __forceinline__ SegChunk seg_chunk_of(const SegWalk& w, int c, const DecodeArgs& a,
                                                 const int32_t* __restrict__ chunks, int num_chunks,
                                                 int num_members, int num_seqs) {
  if (num_chunks <= 32) {
    return SegChunk{__shfl_sync(kFull, w.cl.leader, c), __shfl_sync(kFull, w.cl.moff, c),
                    __shfl_sync(kFull, w.cl.mcount, c), __shfl_sync(kFull, w.cl.ns, c)};
  }
  return seg_chunk(a, chunks, c, num_members, num_seqs, false, w.vt);
}

// Lane (kv head, chunk), unit offset within the lane and the lane's steps of
// shared unit u (warp-collective; u < H_kv * s_sh).
__device__ __forceinline__ void seg_locate(const SegWalk& w, int u, const DecodeArgs& a,
                                           const int32_t* __restrict__ chunks, int num_chunks, int num_members,
                                           int num_seqs, int& kvh, int& c, int& off, int& ns) {
  const int lane = threadIdx.x & 31;
  kvh = u / w.s_sh;
  int r = u - kvh * w.s_sh;
  c = 0;
  off = 0;
  ns = 0;
  for (int c0 = 0; c0 < num_chunks; c0 += 32) {
    int n, incl;
    if (num_chunks <= 32) {
      n = seg_lane_units(w.cl.ns);
      incl = w.cl_incl;
    } else {
      const int cc = c0 + lane;
      n = cc < num_chunks ? seg_lane_units(seg_chunk(a, chunks, cc, num_members, num_seqs, false, w.vt).ns) : 0;
      incl = warp_incl_sum(n);
    }
    const uint32_t hit = __ballot_sync(kFull, incl > r);
    if (hit) {
      const int l = __ffs(hit) - 1;
      const int nl = __shfl_sync(kFull, n, l);
      c = c0 + l;
      off = r - (__shfl_sync(kFull, incl, l) - nl);
      ns = nl - kSegLeadIn;
      return;
    }
    r -= __shfl_sync(kFull, incl, 31);
  }
}

// Start of CTA k's range: total * k / ctas, except that a range never ends
// inside the steps of a lane of one partition, at most 8 steps (such a cut moves
// to the nearer end of them): such a lane has one slot.
__device__ __forceinline__ int seg_cut(const SegWalk& w, int k, const DecodeArgs& a,
                                       const int32_t* __restrict__ chunks, int num_chunks, int num_members,
                                       int num_seqs) {
  int u = (int)((unsigned)w.total * (unsigned)k / (unsigned)w.ctas);
  if (u < w.base && w.s_sh > 0) {
    int kvh, c, off, ns;
    seg_locate(w, u, a, chunks, num_chunks, num_members, num_seqs, kvh, c, off, ns);
    const int step = off - kSegLeadIn;
    if (ns <= 8 && step > 0) u += 2 * step < ns ? -step : ns - step;
  }
  return u;
}

template <int E>
__device__ __forceinline__ void seg_walk_init(SegWalk& w, const DecodeArgs& a, const int32_t* __restrict__ chunks,
                                              int num_chunks, const int32_t* __restrict__ members, int num_members,
                                              const int32_t* __restrict__ first_partition, int num_seqs,
                                              bool fold_tails, int vt, bool report) {
  const int lane = threadIdx.x & 31;
  w.vt = vt;
  // Shared units per kv head and the tail weight per kv head.  The chunk, member
  // and sequence loads of one pass are independent (one round trip); plans of up
  // to 32 chunks keep their chunks in lane registers.
  if (lane < num_members) asm volatile("prefetch.global.L1 [%0];\n" ::"l"(members + lane));
  int s_sh = 0, tw = 0;
  w.cl = SegChunk{0, 0, 0, 0};
  w.cl_incl = 0;
  for (int i0 = 0; i0 < num_chunks || i0 < num_seqs; i0 += 32) {
    const int i = i0 + lane;
    const SegChunk ci =
        i < num_chunks ? seg_chunk(a, chunks, i, num_members, num_seqs, report, vt) : SegChunk{0, 0, 0, 0};
    const int n = seg_lane_units(ci.ns);
    int T = 0, fp, ctx;
    if (fold_tails) seg_tail_of(a, first_partition, i, num_seqs, T, fp, ctx);
    const int incl = warp_incl_sum(n);
    if (i0 == 0) {
      w.cl = ci;
      w.cl_incl = incl;
    }
    s_sh += __shfl_sync(kFull, incl, 31);
    tw += __shfl_sync(kFull, warp_incl_sum(T > 0 ? T + E : 0), 31);
  }
  w.s_sh = s_sh;
  w.tw = tw;
  w.base = a.num_kv_heads * s_sh;
  w.total = w.base + a.num_kv_heads * tw;
  // Every range spans at least 16 units; CTAs past the last range get none.
  w.ctas = w.total / 16;
  if (w.ctas < 1) w.ctas = 1;
  if (w.ctas > gridDim.x) w.ctas = gridDim.x;
  if ((int)blockIdx.x < w.ctas) {
    w.u0 = seg_cut(w, blockIdx.x, a, chunks, num_chunks, num_members, num_seqs);
    w.u1 = blockIdx.x + 1 == w.ctas ? w.total : seg_cut(w, blockIdx.x + 1, a, chunks, num_chunks, num_members, num_seqs);
  } else {
    w.u0 = w.u1 = w.total;
  }
  // Shared cursor: lane (kv head, chunk) and unit offset of unit u0.
  w.su = w.su_end = 0;
  w.skvh = w.sc = w.soff = 0;
  w.sci = SegChunk{0, 0, 0, 0};
  if (w.u0 < w.base && s_sh > 0) {
    w.su = w.u0;
    w.su_end = w.u1 < w.base ? w.u1 : w.base;
    int ns;
    seg_locate(w, w.u0, a, chunks, num_chunks, num_members, num_seqs, w.skvh, w.sc, w.soff, ns);
    w.sci = seg_chunk_of(w, w.sc, a, chunks, num_chunks, num_members, num_seqs);
  }
  // Tail cursor: the first kv head whose tail lanes can start in [u0, u1).
  w.tdone = !(tw > 0 && w.u1 > w.base && w.u1 > w.u0);
  w.tkvh = (!w.tdone && w.u0 > w.base) ? (w.u0 - w.base) / tw : 0;
  w.tm0 = 0;
  w.tw_at = w.base + w.tkvh * tw;
  w.tmask = 0;
  w.tloaded = false;
  w.tT = w.tfp = w.tctx = 0;
}

template <int E>
__device__ __forceinline__ bool seg_walk_next(SegWalk& w, Seg& s, const DecodeArgs& a,
                                              const int32_t* __restrict__ chunks, int num_chunks,
                                              const int32_t* __restrict__ members, int num_members,
                                              const int32_t* __restrict__ first_partition, int num_seqs) {
  const int lane = threadIdx.x & 31;
  while (w.su < w.su_end) {
    const int units = seg_lane_units(w.sci.ns);
    const int len = w.sci.ns;
    const int lane0 = w.su - w.soff;
    const int off1 = units - w.soff < w.su_end - w.su ? units : w.soff + (w.su_end - w.su);
    const int s0 = max(0, w.soff - kSegLeadIn), s1 = max(0, off1 - kSegLeadIn);
    w.su += off1 - w.soff;
    w.soff = off1;
    const int kvh = w.skvh;
    const SegChunk ci = w.sci;
    if (w.soff == units && w.su < w.su_end) {  // on to the next non-empty lane
      do {
        if (++w.sc == num_chunks) {
          w.sc = 0;
          ++w.skvh;
        }
        w.sci = seg_chunk_of(w, w.sc, a, chunks, num_chunks, num_members, num_seqs);
      } while (w.sci.ns == 0 && w.skvh < a.num_kv_heads);
      w.soff = 0;
    }
    if (s1 <= s0) continue;  // the range held only lead-in units of this lane
    // Slot: 0 for the segment with the lane's first step; a segment that starts
    // after it starts this CTA's range, and the CTAs from the one holding the
    // lane's first step up to this one each began one segment of the lane before.
    int slot = 0;
    if (s0 > 0) {
      const int first = lane0 + kSegLeadIn;
      slot = (int)blockIdx.x - (int)(((unsigned)w.ctas * (unsigned)(first + 1) - 1u) / (unsigned)w.total);
    }
    const int mark_end = s1 == len ? (ci.ns + 7) / 8 : slot + 1;
    // A verify lane reads its leader's whole context, each row up to its own token.
    const int ctx = w.vt > 0 ? context_of(a, ci.leader, false) : INT_MAX;
    const int causal = w.vt > 0 ? w.vt - 1 - (ci.moff - ci.leader * w.vt) : 0;
    const int final = w.vt > 0 && s0 == 0 && s1 == len;
    s = Seg{0, kvh, ci.leader, ci.moff, ci.mcount, -1, s0, s1, ctx, slot, mark_end, causal, final};
    return true;
  }
  while (true) {
    if (w.tmask) {
      const int l = __ffs(w.tmask) - 1;
      w.tmask &= w.tmask - 1;
      const int T = __shfl_sync(kFull, w.tT, l), b = w.tm0 + l;
      const int fp = __shfl_sync(kFull, w.tfp, l), ctx = __shfl_sync(kFull, w.tctx, l);
      s = Seg{1, w.tkvh, b, 0, 1, b, 8 * fp, 8 * fp + T, ctx, fp, (ctx + kPartition - 1) / kPartition, 0, 0};
      return true;
    }
    if (w.tdone) return false;
    if (w.tloaded) {  // the loaded batch is handed out: the next one
      w.tloaded = false;
      w.tm0 += 32;
      if (w.tm0 >= num_seqs) {
        w.tm0 = 0;
        if (++w.tkvh >= a.num_kv_heads) {
          w.tdone = true;
          return false;
        }
      }
    }
    if (w.tw_at >= w.u1) {
      w.tdone = true;
      return false;
    }
    seg_tail_of(a, first_partition, w.tm0 + lane, num_seqs, w.tT, w.tfp, w.tctx);
    const int wt = w.tT > 0 ? w.tT + E : 0;
    const int incl = warp_incl_sum(wt);
    const int start = w.tw_at + incl - wt;
    w.tmask = __ballot_sync(kFull, wt > 0 && start >= w.u0 && start < w.u1);
    w.tw_at += __shfl_sync(kFull, incl, 31);
    w.tloaded = true;
  }
}

// ROWS_OUT: verify launches, whose segments may write their rows' outputs (see Seg).
template <typename T, int D, int STAGES, bool ROWS_OUT>
__global__ void __launch_bounds__(SegShape<D, STAGES>::kThreads, 1)
    decode_shared_seg_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tmap_k,
                             const __grid_constant__ CUtensorMap tmap_v, int tma_k,
                             const int32_t* __restrict__ chunks, int num_chunks,
                             const int32_t* __restrict__ members, int num_members,
                             const int32_t* __restrict__ first_partition, int num_seqs, int fold_tails,
                             int verify_tokens, int wait_at_start, int fault, int32_t* __restrict__ merge_list) {
  using S = SegShape<D, STAGES>;
  constexpr int E = S::kEpilogueSteps;
  extern __shared__ uint8_t smem_raw[];
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int bs = a.block_size;
  const int G = a.group;

  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw);
  // Written by the producers, published with q_full: the segment in buffer b
  // -- [0] valid (0 ends the walk), [1] kv head, [2] s0, [3] s1, [4] rows,
  // [5] context limit, [6] slot, [7] end of the slots marked empty, [8] the
  // sequence whose table gives the pages, [9 + k] bit i: 16-token group k of
  // step s0 + i is on an out-of-range page (i < 32) -- and the workspace row
  // base of each of its query rows (-1: none).
  volatile int32_t* desc = reinterpret_cast<volatile int32_t*>(base_ptr + S::kDescOff);  // [2][16]
  int32_t* prow_s = reinterpret_cast<int32_t*>(base_ptr + S::kRowOff);                   // [2][kRows]
  const uint32_t bar0 = base + S::kBarOff;
  auto s_full = [&](int b) { return bar0 + 8u * b; };
  auto p_full = [&](int b) { return bar0 + 16u + 8u * b; };
  auto o_done = [&](int b) { return bar0 + 32u + 8u * b; };
  auto q_full = [&](int b) { return bar0 + 48u + 8u * b; };
  auto item_free = [&](int b) { return bar0 + 64u + 8u * b; };
  auto kv_full = [&](int st) { return bar0 + 80u + 8u * st; };
  auto kv_empty = [&](int st) { return bar0 + 80u + 8u * STAGES + 8u * st; };
  const uint32_t mma_drain = bar0 + 80u + 16u * STAGES;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base_ptr + S::kTaddrOff + 8);
  const uint32_t taddr_slot = base + S::kTaddrOff;

  auto wait = [&](uint32_t bar, uint32_t parity) -> bool {
    const long long t0 = clock64();
    while (!tc05::mbar_try_wait_sleep(bar, parity, 20000u)) {
      if (*abort_flag) return false;
      if (clock64() - t0 > kWaitCycles) {
        *abort_flag = 1;
        return false;
      }
    }
    return true;
  };
  auto wwait = [&](uint32_t bar, uint32_t parity) -> bool { return __all_sync(kFull, wait(bar, parity)); };

  // The producers' walk of the plan and their first page windows do not touch
  // shared memory: their global loads start before the set-up below.
  const bool producer = warp >= 4 && warp != S::kMmaWarp;
  const int pw = producer ? S::producer_of(warp) : 0;  // group pw of every step; query rows 32 pw + lane
  SegWalk walk;
  Seg seg, nxt;
  bool have = false, have_nxt = false;
  // Page of group pw of step w0 + lane of segment s, -1 outside the segment or the table.
  auto window = [&](const Seg& s, int w0) -> int {
    const int64_t tok = 64 * (int64_t)(w0 + lane) + 16 * pw;
    const int64_t blk = tok / bs;
    return (w0 + lane < s.s1 && tok < s.ctx && blk < a.max_blocks_per_seq)
               ? __ldg(a.block_tables + (int64_t)s.leader * a.max_blocks_per_seq + blk)
               : -1;
  };
  auto next_seg = [&](Seg& s) {
    return seg_walk_next<E>(walk, s, a, chunks, num_chunks, members, num_members, first_partition, num_seqs);
  };
  // The segment after the current one is known, and its first page windows are
  // requested, as soon as the current one starts: its query rows are loaded
  // three steps before the current one ends without waiting for the table.
  int win_cur = -1, win_nxt = -1, nxt_cur = -1, nxt_nxt = -1;
  if (producer) {
    // Launched as a programmatic dependent of an arbitrary kernel: nothing is read
    // before that grid has finished (its launch and the set-up below overlap it).
    // Every global write of this grid follows a producer's load, hence this wait.
    if (wait_at_start) {
      // The plan and the lengths into L2 meanwhile (a prefetch returns nothing to
      // the thread, and L2 holds any later write of the grid before, so this is
      // safe whatever that grid writes): the walk's first loads then hit L2.
      const int32_t* arr = pw == 0 ? chunks : pw == 1 ? members : pw == 2 ? first_partition : a.context_lens;
      const int64_t words = pw == 0 ? 4 * (int64_t)num_chunks : pw == 1 ? num_members : num_seqs;
      if (arr != nullptr && 32 * (int64_t)lane < words)
        asm volatile("prefetch.global.L2 [%0];\n" ::"l"(arr + 32 * (int64_t)lane));
      asm volatile("griddepcontrol.wait;\n" ::: "memory");
    }
    seg_walk_init<E>(walk, a, chunks, num_chunks, members, num_members, first_partition, num_seqs, fold_tails != 0,
                     verify_tokens, pw == 0 && lane == 0 && blockIdx.x == 0);
    have = next_seg(seg);
    if (have) {
      win_cur = window(seg, seg.s0);
      win_nxt = window(seg, seg.s0 + 32);
    }
    have_nxt = have && next_seg(nxt);
    nxt_cur = have_nxt ? window(nxt, nxt.s0) : -1;
    nxt_nxt = have_nxt ? window(nxt, nxt.s0 + 32) : -1;
  }

  // -- set-up -----------------------------------------------------------------------------------
  if (tid == 0) {
    for (int b = 0; b < 2; ++b) {
      tc05::mbar_init(s_full(b), 1);
      tc05::mbar_init(p_full(b), 4);
      tc05::mbar_init(o_done(b), 1);
      tc05::mbar_init(q_full(b), S::kProducerWarps);  // lane 0 of each producer warp (+ their copies)
      tc05::mbar_init(item_free(b), 4);
    }
    for (int st = 0; st < STAGES; ++st) {
      tc05::mbar_init(kv_full(st), S::kProducerWarps);
      tc05::mbar_init(kv_empty(st), 1);
    }
    tc05::mbar_init(mma_drain, 1);
    *abort_flag = 0;
    tc05::fence_mbar_init();
    if (tma_k) {
      tc05::prefetch_tensormap(&tmap_k);
      tc05::prefetch_tensormap(&tmap_v);
    }
  }
  if (warp == 0) {
    tc05::alloc(taddr_slot, S::kTmemCols);
    tc05::relinquish();
  }
  tc05::fence_before();
  __syncthreads();
  tc05::fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(base_ptr + S::kTaddrOff);

  // The merge that follows may be launched now (it waits for this grid).
  if (tid == 0) asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  if (producer) {
    // ---------------------------------------------------------------- producers
    const T* qbase = reinterpret_cast<const T*>(a.q);
    const T* kcache = reinterpret_cast<const T*>(a.key_cache);
    const T* vcache = reinterpret_cast<const T*>(a.value_cache);
    // Query rows of segment s into buffer qb, its workspace row bases, and its
    // descriptor (producer pw: the out-of-range pages of group pw in the first 32
    // steps, from `win`); q_full(qb) completes once every producer has arrived and
    // the copies have landed.
    auto load_q = [&](const Seg& s, int qb, int win) {
      {
        const uint32_t qs = base + S::kQOff + qb * S::kQBytes;
        const int r = pw * 32 + lane;
        const int nrows = s.mcount * G;
        int64_t row = -1;
        if (r < nrows) {
          const int mi = r / G;
          const int b = s.kind == 0 ? __ldg(members + s.moff + mi) : s.b;
          if ((unsigned)b < (unsigned)num_seqs) row = (int64_t)b * a.num_q_heads + s.kvh * G + (r - mi * G);
          else flag_status(a.status, PA_DEV_BAD_PLAN);
        }
        const T* src = qbase + (row < 0 ? 0 : row) * D;
#pragma unroll
        for (int ck = 0; ck < D / 8; ++ck)
          cp_async_16(qs + (ck >> 3) * S::kQBlockBytes + r * 128 + (((ck & 7) ^ (r & 7)) << 4), src + ck * 8,
                      row < 0 ? 0u : 16u);
        prow_s[qb * S::kRows + r] = row < 0 ? -1 : (int32_t)(row * a.max_partitions);
        tc05::cp_async_arrive(q_full(qb));
        const int64_t tok = 64 * (int64_t)(s.s0 + lane) + 16 * pw;
        const uint32_t bad = __ballot_sync(kFull, s.s0 + lane < s.s1 && tok < s.ctx &&
                                                      (unsigned)win >= (unsigned)a.num_blocks);
        if (lane == 0) desc[qb * 16 + 9 + pw] = (int32_t)bad;
        if (pw == 0 && lane == 0) {
          desc[qb * 16 + 1] = s.kvh;
          desc[qb * 16 + 2] = s.s0;
          desc[qb * 16 + 3] = s.s1;
          desc[qb * 16 + 4] = nrows;
          desc[qb * 16 + 5] = s.ctx;
          desc[qb * 16 + 6] = s.slot;
          desc[qb * 16 + 7] = s.mark_end;
          desc[qb * 16 + 8] = s.leader;
          desc[qb * 16 + 13] = s.causal;
          desc[qb * 16 + 14] = s.final;
          desc[qb * 16 + 0] = 1;
        }
      }
    };
    auto end_walk = [&](int qb) {  // buffer qb holds no segment: the other roles stop there
      if (pw == 0 && lane == 0) desc[qb * 16 + 0] = 0;
    };
    auto publish_q = [&](int qb) {
      __syncwarp();
      if (lane == 0) tc05::mbar_arrive(q_full(qb));
    };
    if (have) load_q(seg, 0, win_cur);
    else end_walk(0);
    if (fault != PA_FAULT_WITHHOLD_FIRST_ITEM) publish_q(0);  // test hook: the other roles' waits run out
    int64_t g = 0;
    bool stop = false;
    for (int j = 0; have && !stop; ++j) {
      const int qb = j & 1;
      const int len = seg.s1 - seg.s0;
      const int qload_at = len > 3 ? len - 3 : 0;
      int w0 = seg.s0;
      for (int i = 0; i < len; ++i, ++g) {
        const int step = seg.s0 + i;
        if (step - w0 == 32) {
          w0 += 32;
          win_cur = win_nxt;
          win_nxt = window(seg, w0 + 32);
        }
        const int st = (int)(g % STAGES);
        if (g >= STAGES && !wwait(kv_empty(st), (uint32_t)(((g - STAGES) / STAGES) & 1))) { stop = true; break; }
        const int page = __shfl_sync(kFull, win_cur, step - w0);
        const int tok = 64 * step + 16 * pw;
        const bool page_ok = (unsigned)page < (unsigned)a.num_blocks;
        if (lane == 0 && tok < seg.ctx && !page_ok) flag_status(a.status, PA_DEV_BAD_PAGE);
        const int64_t slab = ((int64_t)(page_ok ? page : 0) * a.num_kv_heads + seg.kvh) * bs + tok % bs;
        const uint32_t stage = base + S::kStageOff + st * S::kStageBytes;
        // V by the tensor map too when the whole group lies in the context (or the
        // page is out of range: the box then starts past the tensor and loads zeros);
        // a group the context ends inside needs zeros in its later rows, since a
        // weight of 0 times a stale slot's NaN would still reach O.
        const bool tma_v = tma_k && (!page_ok || tok + 16 <= seg.ctx);
        // The rest (V of such a group, and K and V without the tensor maps): 16-byte
        // cp.async copies, zero past the context and on an out-of-range page; their
        // completion joins the stage's phase before this warp's arrival below.
#pragma unroll
        for (int kv = 0; kv < 2; ++kv) {
          if (kv == 0 ? tma_k : tma_v) continue;
          const T* cache = kv ? vcache : kcache;
#pragma unroll
          for (int i2 = 0; i2 < S::kCopiesPerGroup; ++i2) {
            const int rl = i2 * S::kRowsPerCopy + lane / S::kChunksPerRow;  // row within the group
            const int ck = lane % S::kChunksPerRow;
            const int row = 16 * pw + rl;                                    // row within the step
            const bool valid = page_ok && tok + rl < seg.ctx;
            const T* src = cache + (valid ? (slab + rl) * D + ck * 8 : 0);
            const uint32_t dst = stage + kv * S::kTileBytes + (ck >> 3) * S::kKVBlockBytes + row * 128 +
                                 (((ck & 7) ^ (row & 7)) << 4);
            cp_async_16(dst, src, valid ? 16u : 0u);
          }
        }
        tc05::cp_async_arrive(kv_full(st));
        __syncwarp();
        if (lane == 0) {
          if (tma_k) {
            // K by the tensor-memory-access unit: one 16-row box per 64-column block
            // (an out-of-range page loads as zeros; rows past the context are masked
            // by the softmax).  The arrival announces the bytes before the copies start.
            tc05::mbar_arrive_expect_tx(kv_full(st), (tma_v ? 2 : 1) * S::kBlocks * 16 * 128);
            const int32_t y = page_ok ? (int32_t)slab : (int32_t)((int64_t)a.num_blocks * a.num_kv_heads * bs);
#pragma unroll
            for (int blk = 0; blk < S::kBlocks; ++blk)
              tc05::tma_load_2d(stage + blk * S::kKVBlockBytes + 16 * pw * 128, &tmap_k, kv_full(st), 64 * blk, y);
            if (tma_v) {
#pragma unroll
              for (int blk = 0; blk < S::kBlocks; ++blk)
                tc05::tma_load_2d(stage + S::kTileBytes + blk * S::kKVBlockBytes + 16 * pw * 128, &tmap_v,
                                  kv_full(st), 64 * blk, y);
            }
          } else {
            tc05::mbar_arrive(kv_full(st));
          }
        }
        // Three steps before the end: the next segment's queries go into the other
        // buffer once the segment that last used it (j - 1) has been read out.
        if (i == qload_at) {
          if (j >= 1 && !wwait(item_free(qb ^ 1), (uint32_t)(((j - 1) >> 1) & 1))) { stop = true; break; }
          if (have_nxt) load_q(nxt, qb ^ 1, nxt_cur);
          else end_walk(qb ^ 1);
          publish_q(qb ^ 1);
        }
      }
      if (stop || __any_sync(kFull, *abort_flag != 0)) break;
      seg = nxt;
      have = have_nxt;
      win_cur = nxt_cur;
      win_nxt = nxt_nxt;
      have_nxt = have && next_seg(nxt);
      nxt_cur = have_nxt ? window(nxt, nxt.s0) : -1;
      nxt_nxt = have_nxt ? window(nxt, nxt.s0 + 32) : -1;
    }
    tc05::cp_async_wait_all();  // nothing may land in shared memory after the CTA leaves
  } else if (warp == S::kMmaWarp) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t fmt = std::is_same<T, __nv_bfloat16>::value ? 1u : 0u;
      constexpr uint32_t idesc_s = tc05::instr_desc_f16(fmt, S::kRows, S::kStep, 0, 0);
      constexpr uint32_t idesc_o = tc05::instr_desc_f16(fmt, S::kRows, D, 0, 1);
      auto mma2 = [&](int64_t gp, int j, bool first) -> bool {  // O[segment j] (+)= P(gp) . V(gp)
        if (!wait(p_full((int)(gp & 1)), (uint32_t)((gp >> 1) & 1))) return false;
        tc05::fence_after();
        const int st = (int)(gp % STAGES);
        const uint32_t vs = base + S::kStageOff + st * S::kStageBytes + S::kTileBytes;
        const uint32_t ocol = S::kOCol + 128u * (uint32_t)(j & 1);
#pragma unroll
        for (int kt = 0; kt < S::kStep / 16; ++kt)
          tc05::mma_ts(tmem + ocol, tmem + S::kPCol + 32 * (uint32_t)(gp & 1) + 8 * kt,
                       tc05::smem_desc_sw128(vs + kt * 16 * 128, S::kKVBlockBytes, 1024), idesc_o,
                       (!first || kt > 0) ? 1u : 0u);
        tc05::commit(o_done((int)(gp & 1)));
        tc05::commit(kv_empty(st));
        return true;
      };
      int64_t g = 0;
      bool ok = true;
      for (int j = 0; ok; ++j) {
        const int qb = j & 1;
        if (!wait(q_full(qb), (uint32_t)((j >> 1) & 1))) break;
        if (desc[qb * 16 + 0] == 0) break;  // the walk has ended
        const int len = desc[qb * 16 + 3] - desc[qb * 16 + 2];
        tc05::fence_after();
        tc05::fence_proxy_async_smem();
        const uint32_t qs = base + S::kQOff + qb * S::kQBytes;
        for (int i = 0; i < len; ++i, ++g) {
          const int st = (int)(g % STAGES);
          // S buffer g & 1 is free: this thread has seen p_full(g - 2), which the softmax
          // raises after reading S(g - 2).
          if (!wait(kv_full(st), (uint32_t)((g / STAGES) & 1))) { ok = false; break; }
          tc05::fence_after();
          tc05::fence_proxy_async_smem();  // the stage's cp.async writes, for the tensor cores
          const uint32_t ks = base + S::kStageOff + st * S::kStageBytes;
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t blk = k >> 2, koff = (k & 3) * 32;
            tc05::mma_ss(tmem + S::kSCol + 64 * (uint32_t)(g & 1),
                         tc05::smem_desc_sw128(qs + blk * S::kQBlockBytes + koff, 16, 1024),
                         tc05::smem_desc_sw128(ks + blk * S::kKVBlockBytes + koff, 16, 1024), idesc_s,
                         k > 0 ? 1u : 0u);
          }
          tc05::commit(s_full((int)(g & 1)));
          if (i >= 1 && !mma2(g - 1, j, i == 1)) { ok = false; break; }
        }
        // Close the segment (its epilogue must not wait for the next segment's queries).
        if (ok && !mma2(g - 1, j, len == 1)) ok = false;
      }
      tc05::commit(mma_drain);
      {
        const long long t0 = clock64();
        while (!tc05::mbar_try_wait(mma_drain, 0) && clock64() - t0 < kWaitCycles) {
        }
      }
    }
  } else {
    // ---------------------------------------------------------------- softmax warps 0-3
    const uint32_t row_t = tmem + ((uint32_t)(32 * warp) << 16);
    int64_t g = 0;
    for (int j = 0;; ++j) {
      const int qb = j & 1;
      if (!wwait(q_full(qb), (uint32_t)((j >> 1) & 1))) break;  // segment, rows and descriptor
      if (desc[qb * 16 + 0] == 0) break;                          // the walk has ended
      const int s0 = desc[qb * 16 + 2], s1 = desc[qb * 16 + 3];
      const int nrows = desc[qb * 16 + 4], ctx = desc[qb * 16 + 5];
      const int slot = desc[qb * 16 + 6], mark_end = desc[qb * 16 + 7], leader = desc[qb * 16 + 8];
      // This thread's row sees the tokens before ctx_row (its own causal limit).
      const int ctx_row = ctx - max(0, desc[qb * 16 + 13] - (32 * warp + lane) / a.group);
      const bool busy = 32 * warp < nrows;
      // Out-of-range pages: bit i of bad_w[k] is group k of step mw0 + i.  The
      // producers publish the first 32 steps; later windows of 32 steps are
      // requested one window ahead (page of group k of step mw0 + 32 + lane).
      uint32_t bad_w[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) bad_w[q] = (uint32_t)desc[qb * 16 + 9 + q];
      int mw0 = s0;
      int pre[4];
      auto request = [&](int w0) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int st_ = w0 + lane;
          const int64_t tok = 64 * (int64_t)st_ + 16 * q;
          const int64_t blk = tok / bs;
          pre[q] = (st_ < s1 && tok < ctx && blk < a.max_blocks_per_seq)
                       ? __ldg(a.block_tables + (int64_t)leader * a.max_blocks_per_seq + blk)
                       : 0;
        }
      };
      if (s1 > s0 + 32) request(s0 + 32);
      float m_use = -INFINITY, l = 0.f;
      bool ok = true;
      for (int step = s0; step < s1; ++step, ++g) {
        if (step == mw0 + 32) {
#pragma unroll
          for (int q = 0; q < 4; ++q) bad_w[q] = __ballot_sync(kFull, (unsigned)pre[q] >= (unsigned)a.num_blocks);
          mw0 += 32;
          if (s1 > mw0 + 32) request(mw0 + 32);
        }
        if (!wwait(s_full((int)(g & 1)), (uint32_t)((g >> 1) & 1))) { ok = false; break; }
        tc05::fence_after();
        uint32_t sreg[2][32];
        if (busy) {
          tc05::ld32(row_t + S::kSCol + 64 * (uint32_t)(g & 1), sreg[0]);
          tc05::ld32(row_t + S::kSCol + 64 * (uint32_t)(g & 1) + 32, sreg[1]);
          tc05::wait_ld();
        }
        const int sh = step - mw0;
        const int bad = (int)(((bad_w[0] >> sh) & 1u) | (((bad_w[1] >> sh) & 1u) << 1) |
                              (((bad_w[2] >> sh) & 1u) << 2) | (((bad_w[3] >> sh) & 1u) << 3));
        const int lim = ctx_row - 64 * step;  // tokens of this step this row sees
        uint32_t pk[32];
        float alpha = 1.f;
        if (busy) {
          float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
          float nref;
          if (bad == 0 && lim >= 64 && a.qk_scale_log2 > 0.f) {
#pragma unroll
            for (int e = 0; e < 64; ++e) mx4[e & 3] = fmaxf(mx4[e & 3], __uint_as_float(sreg[e >> 5][e & 31]));
            const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * a.qk_scale_log2;
            if (mx > m_use + 8.f) {
              alpha = m_use == -INFINITY ? 0.f : ex2_approx(m_use - mx);
              m_use = mx;
            }
            nref = -m_use;
            float ls[4] = {0.f, 0.f, 0.f, 0.f};
            // Every score is finite here: half the weights on the special-function
            // unit, half on the FMA pipe, which the softmax otherwise leaves idle.
#pragma unroll
            for (int jj = 0; jj < 32; ++jj) {
              const int e0 = 2 * jj, e1 = 2 * jj + 1;
              const float p0 = ex2_approx(fmaf(__uint_as_float(sreg[e0 >> 5][e0 & 31]), a.qk_scale_log2, nref));
              const float p1 = exp2_poly(fmaf(__uint_as_float(sreg[e1 >> 5][e1 & 31]), a.qk_scale_log2, nref));
              ls[jj & 3] += p0 + p1;
              pk[jj] = pack2<T>(p0, p1);
            }
            l = l * alpha + ((ls[0] + ls[1]) + (ls[2] + ls[3]));
          } else {
            // Tokens past the context or on an out-of-range page have score -inf (weight 0).
#pragma unroll
            for (int e = 0; e < 64; ++e) {
              const bool masked = e >= lim || ((bad >> (e >> 4)) & 1);
              const float v = masked ? -INFINITY : __uint_as_float(sreg[e >> 5][e & 31]) * a.qk_scale_log2;
              sreg[e >> 5][e & 31] = __float_as_uint(v);
              mx4[e & 3] = fmaxf(mx4[e & 3], v);
            }
            const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
            if (mx > m_use + 8.f) {
              alpha = m_use == -INFINITY ? 0.f : ex2_approx(m_use - mx);
              m_use = mx;
            }
            nref = m_use == -INFINITY ? 0.f : -m_use;
            float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int jj = 0; jj < 32; ++jj) {
              const int e0 = 2 * jj, e1 = 2 * jj + 1;
              const float p0 = ex2_approx(__uint_as_float(sreg[e0 >> 5][e0 & 31]) + nref);
              const float p1 = ex2_approx(__uint_as_float(sreg[e1 >> 5][e1 & 31]) + nref);
              ls[jj & 3] += p0 + p1;
              pk[jj] = pack2<T>(p0, p1);
            }
            l = l * alpha + ((ls[0] + ls[1]) + (ls[2] + ls[3]));
          }
        }
        if (busy && step > s0 && __any_sync(kFull, alpha != 1.f)) {
          // O is current once O += P.V of step g - 1 has completed.
          if (!wwait(o_done((int)((g - 1) & 1)), (uint32_t)(((g - 1) >> 1) & 1))) { ok = false; break; }
          tc05::fence_after();
          const uint32_t ocol = S::kOCol + 128u * (uint32_t)qb;
#pragma unroll 1
          for (int cb = 0; cb < D / 16; ++cb) {
            uint32_t ov[16];
            tc05::ld16(row_t + ocol + 16 * cb, ov);
            tc05::wait_ld();
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) ov[jj] = __float_as_uint(__uint_as_float(ov[jj]) * alpha);
            tc05::st16(row_t + ocol + 16 * cb, ov);
          }
        }
        // P buffer g & 1 was last read by O += P.V of step g - 2, which the MMA
        // thread issued before S(g): S(g) has completed, so that MMA has too.
        if (busy) {
          tc05::st32(row_t + S::kPCol + 32 * (uint32_t)(g & 1), pk);
          tc05::wait_st();
        }
        tc05::fence_before();
        __syncwarp();
        if (lane == 0) tc05::mbar_arrive(p_full((int)(g & 1)));
      }
      if (!ok) break;
      // Epilogue: the segment's last O += P.V (step g - 1) has to complete.
      const int64_t gl = g - 1;
      if (!wwait(o_done((int)(gl & 1)), (uint32_t)((gl >> 1) & 1))) break;
      tc05::fence_after();
      if (busy) {
        const int32_t rbase = prow_s[qb * S::kRows + tid];  // workspace row base of this thread's query row
        const int32_t prow = rbase < 0 ? -1 : rbase + slot;
        const bool final = ROWS_OUT && desc[qb * 16 + 14] != 0;  // the outputs themselves (see Seg)
        const int32_t orow = rbase < 0 ? -1 : rbase / a.max_partitions;
        const float inv = l > 0.f ? 1.f / l : 0.f;
        if constexpr (ROWS_OUT) {
          // The first run of a lane that other runs continue lists its rows for the
          // merge (which then covers those rows only).
          if (!final && slot == 0 && merge_list != nullptr) {
            const unsigned want = __ballot_sync(kFull, prow >= 0);
            int first = 0;
            if (lane == 0 && want) first = atomicAdd(merge_list, __popc(want));
            first = __shfl_sync(kFull, first, 0);
            if (prow >= 0) merge_list[1 + first + __popc(want & ((1u << lane) - 1u))] = orow;
          }
        }
        const uint32_t ocol = S::kOCol + 128u * (uint32_t)qb;
        constexpr int kTileStride = 20;  // floats
        float* tile = reinterpret_cast<float*>(base_ptr + S::kQOff + qb * S::kQBytes) + warp * 32 * kTileStride;
        float4* wr = reinterpret_cast<float4*>(tile + lane * kTileStride);
        const int rsub = lane >> 2, csub = lane & 3;
#pragma unroll 1
        for (int cb = 0; cb < D / 16; ++cb) {
          uint32_t ov[16];
          tc05::ld16(row_t + ocol + 16 * cb, ov);
          tc05::wait_ld();
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4)
            wr[q4] = make_float4(__uint_as_float(ov[4 * q4]) * inv, __uint_as_float(ov[4 * q4 + 1]) * inv,
                                 __uint_as_float(ov[4 * q4 + 2]) * inv, __uint_as_float(ov[4 * q4 + 3]) * inv);
          __syncwarp();
          float4 v[4];
          int32_t pr[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            pr[i] = __shfl_sync(kFull, final ? orow : prow, 8 * i + rsub);
            v[i] = *reinterpret_cast<const float4*>(tile + (8 * i + rsub) * kTileStride + 4 * csub);
          }
          __syncwarp();
          if (ROWS_OUT && final) {
#pragma unroll
            for (int i = 0; i < 4; ++i)
              if (pr[i] >= 0)
                *reinterpret_cast<uint2*>(reinterpret_cast<T*>(a.out) + (int64_t)pr[i] * D + 16 * cb + 4 * csub) =
                    make_uint2(pack2<T>(v[i].x, v[i].y), pack2<T>(v[i].z, v[i].w));
          } else {
#pragma unroll
            for (int i = 0; i < 4; ++i)
              if (pr[i] >= 0) *reinterpret_cast<float4*>(a.o_part + (int64_t)pr[i] * D + 16 * cb + 4 * csub) = v[i];
          }
        }
        if (ROWS_OUT && final) {
          if (prow >= 0) a.l_part[prow] = -1.f;  // slot 0: this row is done
        } else if (prow >= 0) {
          a.m_part[prow] = m_use == -INFINITY ? -INFINITY : m_use * kLn2;
          a.l_part[prow] = l;
          for (int p = slot + 1; p < mark_end; ++p) {  // the lane's slots no segment takes: empty
            a.m_part[rbase + p] = -INFINITY;
            a.l_part[rbase + p] = 0.f;
          }
        }
      }
      tc05::fence_before();
      __syncwarp();
      if (lane == 0) tc05::mbar_arrive(item_free(qb));
    }
  }

  // -- teardown ---------------------------------------------------------------------------------
  __syncthreads();
  if (*abort_flag && tid == 0) flag_status(a.status, PA_DEV_TIMEOUT);
  tc05::fence_before();
  __syncthreads();
  if (warp == 0) {
    tc05::fence_after();
    tc05::dealloc(tmem, S::kTmemCols);
  }
  // A per-sequence kernel launched before this one (for sequences outside every
  // group) has to finish before this grid does, for the merge that follows.
  if (tid == 0) asm volatile("griddepcontrol.wait;\n" ::: "memory");
}

// ---------------------------------------------------------------------------
// Two-CTAs-per-SM variant of the persistent tcgen05 shared-prefix kernel.  The
// one-CTA kernel is bound by its own per-step chain (S MMA, softmax pass, O
// MMA) while the SM's tensor pipe and its share of DRAM stay mostly idle; two
// CTAs per SM run two such chains side by side.  To fit two per SM a CTA keeps
// one query buffer, a STAGES-deep K/V ring (about 99 KB of shared memory at
// D 128), 256 TMEM columns (S, two P buffers, O) and 7 warps:
//   warps 0-3  softmax, as in the one-CTA kernel; the S row is read in two
//              32-column halves, once for the maximum and once for the
//              weights, to stay within the register budget of two CTAs
//   warps 4-5  producers: 8 TMA boxes each per step; after an item's last step
//              and once its epilogue has freed the query buffer, the next
//              item's queries (two rows per lane), table slice, descriptor and
//              workspace rows
//   warp 6     MMA issuer (one lane): S(g) once the softmax has read S(g-1) out,
//              then O += P(g-1).V(g-1)
// Hand-offs, bounded waits, the abort path and the fault hook are those of the
// one-CTA kernel.
// ---------------------------------------------------------------------------
template <int D, int STAGES>
struct Tc05dShape {
  static constexpr int kProducerWarps = 2;
  static constexpr int kMmaWarp = 6;
  static constexpr int kThreads = 32 * 7;
  static constexpr int kRows = 128;
  static constexpr int kStep = 64;
  static constexpr int kStepsPerItem = kPartition / kStep;  // 8
  static constexpr int kBlocks = D / 64;
  static constexpr int kQBlockBytes = kRows * 128;
  static constexpr int kQBytes = kBlocks * kQBlockBytes;
  static constexpr int kKVBlockBytes = kStep * 128;
  static constexpr int kTileBytes = kBlocks * kKVBlockBytes;
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kBoxBytes = 16 * 128;
  static constexpr int kBoxesPerStep = 2 * (kStep / 16) * kBlocks;
  static constexpr int kBoxesPerWarp = kBoxesPerStep / kProducerWarps;
  static constexpr int kQOff = 0;
  static constexpr int kStageOff = kQBytes;
  static constexpr int kSliceOff = kStageOff + STAGES * kStageBytes;  // int32 [32] table slice
  static constexpr int kDescOff = kSliceOff + 128;                     // int32 [4] item descriptor
  static constexpr int kRowOff = kDescOff + 16;                        // int32 [kRows] workspace rows
  static constexpr int kBarOff = kRowOff + kRows * 4;
  // s_full, s_free, q_full, item_free, mma_drain; p_full, o_done x2; kv_full, kv_empty x STAGES
  static constexpr int kNumBars = 5 + 4 + 2 * STAGES;
  static constexpr int kTaddrOff = kBarOff + 8 * kNumBars;
  static constexpr int kSmemBytes = kTaddrOff + 16 + 1024;
  static constexpr uint32_t kTmemCols = 256;
  static constexpr uint32_t kSCol = 0, kPCol = 64, kOCol = 128;  // S at 0, P[b] at 64 + 32b, O at 128
  static_assert(D <= 128, "O needs D <= 128 columns");
  static_assert(kBoxesPerStep % kProducerWarps == 0 && kBoxesPerWarp <= 32, "one lane per box");
  static_assert(kRows == 2 * 32 * kProducerWarps, "two query rows per producer lane");
  static_assert(kQBytes >= 4 * 32 * 20 * 4, "the epilogue's four 32-row float tiles fit in the query buffer");
  static_assert(2 * (kSmemBytes + 1024) <= 228 * 1024, "two CTAs per SM");
};

template <typename T, int D, int STAGES>
__global__ void __launch_bounds__(Tc05dShape<D, STAGES>::kThreads, 2)
    decode_shared_tc05d_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tmap_k,
                               const __grid_constant__ CUtensorMap tmap_v, const int32_t* __restrict__ chunks,
                               int num_chunks, const int32_t* __restrict__ members, int num_members, int num_seqs,
                               int max_shared_partitions, int fault) {
  using S = Tc05dShape<D, STAGES>;
  constexpr int SPI = S::kStepsPerItem;
  extern __shared__ uint8_t smem_raw[];
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int bs = a.block_size;
  const int G = a.group;
  const int64_t total_rows = (int64_t)a.num_blocks * a.num_kv_heads * bs;
  const int64_t total_items = (int64_t)max_shared_partitions * a.num_kv_heads * num_chunks;

  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw);
  int32_t* tslice = reinterpret_cast<int32_t*>(base_ptr + S::kSliceOff);
  volatile int32_t* desc = reinterpret_cast<volatile int32_t*>(base_ptr + S::kDescOff);
  int32_t* prow_s = reinterpret_cast<int32_t*>(base_ptr + S::kRowOff);
  const uint32_t bar0 = base + S::kBarOff;
  const uint32_t s_full = bar0, s_free = bar0 + 8u, q_full = bar0 + 16u, item_free = bar0 + 24u,
                 mma_drain = bar0 + 32u;
  auto p_full = [&](int b) { return bar0 + 40u + 8u * b; };
  auto o_done = [&](int b) { return bar0 + 56u + 8u * b; };
  auto kv_full = [&](int st) { return bar0 + 72u + 8u * st; };
  auto kv_empty = [&](int st) { return bar0 + 72u + 8u * STAGES + 8u * st; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base_ptr + S::kTaddrOff + 8);
  const uint32_t taddr_slot = base + S::kTaddrOff;

  auto wait = [&](uint32_t bar, uint32_t parity) -> bool {
    const long long t0 = clock64();
    while (!tc05::mbar_try_wait_sleep(bar, parity, 20000u)) {
      if (*abort_flag) return false;
      if (clock64() - t0 > kWaitCycles) {
        *abort_flag = 1;
        return false;
      }
    }
    return true;
  };
  auto wwait = [&](uint32_t bar, uint32_t parity) -> bool { return __all_sync(kFull, wait(bar, parity)); };

  if (tid == 0) {
    tc05::mbar_init(s_full, 1);
    tc05::mbar_init(s_free, 4);      // one arrival per softmax warp
    tc05::mbar_init(q_full, S::kProducerWarps);
    tc05::mbar_init(item_free, 4);
    tc05::mbar_init(mma_drain, 1);
    for (int b = 0; b < 2; ++b) {
      tc05::mbar_init(p_full(b), 4);
      tc05::mbar_init(o_done(b), 1);
    }
    for (int st = 0; st < STAGES; ++st) {
      tc05::mbar_init(kv_full(st), S::kProducerWarps);
      tc05::mbar_init(kv_empty(st), 1);
    }
    *abort_flag = 0;
    tc05::fence_mbar_init();
    tc05::prefetch_tensormap(&tmap_k);
    tc05::prefetch_tensormap(&tmap_v);
  }
  if (warp == 0) {
    tc05::alloc(taddr_slot, S::kTmemCols);
    tc05::relinquish();
  }
  tc05::fence_before();
  __syncthreads();
  tc05::fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(base_ptr + S::kTaddrOff);
  if (tid == 0) asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  int64_t cursor = blockIdx.x;
  int64_t prod_g = 0;
  const uint32_t qs = base + S::kQOff;

  if (warp == 4 || warp == 5) {
    // ---------------------------------------------------------------- producers
    const int pw = warp - 4;
    const T* qbase = reinterpret_cast<const T*>(a.q);
    auto load_pages = [&](const SharedItem& it) -> int {
      const int fb = it.p * kPartition / bs;
      const int nblk = (it.p * kPartition + kPartition - 1) / bs - fb + 1;
      return lane < nblk ? __ldg(a.block_tables + (int64_t)it.leader * a.max_blocks_per_seq + fb + lane) : -1;
    };
    auto load_q = [&](const SharedItem& it, int pages) {
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int r = pw * 64 + 32 * k + lane;
        int64_t row = -1;
        if (r < it.mcount * G) {
          const int mi = r / G;
          const int b = __ldg(members + it.moff + mi);
          if ((unsigned)b < (unsigned)num_seqs) row = (int64_t)b * a.num_q_heads + it.kvh * G + (r - mi * G);
        }
        const T* src = qbase + (row < 0 ? 0 : row) * D;
#pragma unroll
        for (int ck = 0; ck < D / 8; ++ck)
          cp_async_16(qs + (ck >> 3) * S::kQBlockBytes + r * 128 + (((ck & 7) ^ (r & 7)) << 4), src + ck * 8,
                      row < 0 ? 0u : 16u);
        prow_s[r] = row < 0 ? -1 : (int32_t)(row * a.max_partitions + it.p);
      }
      if (pw == 0) {
        tslice[lane] = pages;
        if (lane == 0) {
          desc[1] = it.p;
          desc[2] = it.kvh;
          desc[3] = it.mcount;
          desc[0] = 1;
        }
      }
      cp_async_commit();
    };
    auto end_walk = [&]() {
      if (pw == 0 && lane == 0) desc[0] = 0;
    };
    auto publish_q = [&]() {
      cp_async_wait<0>();
      tc05::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(q_full) : "memory");
    };
    SharedItem it = next_shared_item(cursor, total_items, num_chunks, a, chunks, num_members, num_seqs,
                                     pw == 0 && lane == 0);
    int my_page = it.valid ? load_pages(it) : -1;
    if (it.valid) load_q(it, my_page);
    else end_walk();
    if (fault != PA_FAULT_WITHHOLD_FIRST_ITEM) publish_q();
    else cp_async_wait<0>();  // test hook: the other roles' waits for this hand-off run out
    int64_t g = 0;
    for (int j = 0; it.valid; ++j) {
      const SharedItemPrefetch pf = prefetch_shared_item(cursor, total_items, num_chunks, chunks);
      SharedItem nxt{};
      nxt.valid = false;
      const int fb = it.p * kPartition / bs;
      int nxt_page = -1;
      bool stop = false;
      for (int i = 0; i < SPI; ++i, ++g) {
        const int st = (int)(g % STAGES);
        if (g >= STAGES && !wwait(kv_empty(st), (uint32_t)(((g - STAGES) / STAGES) & 1))) { stop = true; break; }
        if (lane == 0) tc05::mbar_arrive_expect_tx(kv_full(st), S::kBoxesPerWarp * S::kBoxBytes);
        const int box = pw * S::kBoxesPerWarp + lane;
        const int kv = box & 1;
        const int blk = (box >> 1) % S::kBlocks;
        const int rb = ((box >> 1) / S::kBlocks) % (S::kStep / 16);
        const int tok = it.p * kPartition + i * S::kStep + 16 * rb;
        const int page = __shfl_sync(kFull, my_page, tok / bs - fb);
        __syncwarp();
        if (lane < S::kBoxesPerWarp) {
          const int64_t y = (unsigned)page < (unsigned)a.num_blocks
                                ? ((int64_t)page * a.num_kv_heads + it.kvh) * bs + tok % bs
                                : total_rows;  // out of range: the box is filled with zeros
          const uint32_t dst = base + S::kStageOff + st * S::kStageBytes + kv * S::kTileBytes +
                               blk * S::kKVBlockBytes + rb * S::kBoxBytes;
          tc05::tma_load_2d(dst, kv ? (const void*)&tmap_v : (const void*)&tmap_k, kv_full(st), 64 * blk, (int32_t)y);
        }
        __syncwarp();
        prod_g = g + 1;
        if (i == SPI - 3) {
          nxt = resolve_shared_item(pf, cursor, total_items, num_chunks, a, chunks, num_members, num_seqs,
                                    pw == 0 && lane == 0);
          if (nxt.valid) nxt_page = load_pages(nxt);
        }
      }
      if (stop || __any_sync(kFull, *abort_flag != 0)) break;
      // The query buffer is free once item j's epilogue has read it out.
      if (!wwait(item_free, (uint32_t)(j & 1))) break;
      if (nxt.valid) load_q(nxt, nxt_page);
      else end_walk();
      publish_q();
      it = nxt;
      my_page = nxt_page;
    }
    cp_async_wait<0>();  // nothing may land in shared memory after the CTA leaves
  } else if (warp == S::kMmaWarp) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t fmt = std::is_same<T, __nv_bfloat16>::value ? 1u : 0u;
      constexpr uint32_t idesc_s = tc05::instr_desc_f16(fmt, S::kRows, S::kStep, 0, 0);
      constexpr uint32_t idesc_o = tc05::instr_desc_f16(fmt, S::kRows, D, 0, 1);
      auto mma2 = [&](int64_t gp) -> bool {  // O += P(gp) . V(gp)
        if (!wait(p_full((int)(gp & 1)), (uint32_t)((gp >> 1) & 1))) return false;
        tc05::fence_after();
        const int st = (int)(gp % STAGES);
        const uint32_t vs = base + S::kStageOff + st * S::kStageBytes + S::kTileBytes;
        const int ip = (int)(gp % SPI);
#pragma unroll
        for (int kt = 0; kt < S::kStep / 16; ++kt)
          tc05::mma_ts(tmem + S::kOCol, tmem + S::kPCol + 32 * (uint32_t)(gp & 1) + 8 * kt,
                       tc05::smem_desc_sw128(vs + kt * 16 * 128, S::kKVBlockBytes, 1024), idesc_o,
                       (ip > 0 || kt > 0) ? 1u : 0u);
        tc05::commit(o_done((int)(gp & 1)));
        tc05::commit(kv_empty(st));
        return true;
      };
      int64_t g = 0;
      bool ok = true;
      for (int j = 0; ok; ++j) {
        if (!wait(q_full, (uint32_t)(j & 1))) break;
        if (desc[0] == 0) break;  // the walk has ended
        tc05::fence_after();
        tc05::fence_proxy_async_smem();
        for (int i = 0; i < SPI; ++i, ++g) {
          const int st = (int)(g % STAGES);
          if (!wait(kv_full(st), (uint32_t)((g / STAGES) & 1))) { ok = false; break; }
          if (g >= 1 && !wait(s_free, (uint32_t)((g - 1) & 1))) { ok = false; break; }  // S(g-1) read out
          tc05::fence_after();
          const uint32_t ks = base + S::kStageOff + st * S::kStageBytes;
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t blk = k >> 2, koff = (k & 3) * 32;
            tc05::mma_ss(tmem + S::kSCol, tc05::smem_desc_sw128(qs + blk * S::kQBlockBytes + koff, 16, 1024),
                         tc05::smem_desc_sw128(ks + blk * S::kKVBlockBytes + koff, 16, 1024), idesc_s,
                         k > 0 ? 1u : 0u);
          }
          tc05::commit(s_full);
          if (i >= 1 && !mma2(g - 1)) { ok = false; break; }
        }
        if (ok && !mma2(g - 1)) ok = false;  // close the item
      }
      tc05::commit(mma_drain);
      {
        const long long t0 = clock64();
        while (!tc05::mbar_try_wait(mma_drain, 0) && clock64() - t0 < kWaitCycles) {
        }
      }
    }
  } else if (warp < 4) {
    // ---------------------------------------------------------------- softmax warps 0-3
    const uint32_t row_t = tmem + ((uint32_t)(32 * warp) << 16);
    int64_t g = 0;
    for (int j = 0;; ++j) {
      if (!wwait(q_full, (uint32_t)(j & 1))) break;  // item, table slice and rows
      if (desc[0] == 0) break;                        // the walk has ended
      const int ip = desc[1];
      const int mcount = desc[3];
      const bool busy = 32 * warp < mcount * G;
      const uint32_t page_ok = __ballot_sync(
          kFull, (unsigned)tslice[(ip * kPartition + 16 * lane) / bs - ip * kPartition / bs] < (unsigned)a.num_blocks);
      float m_use = -INFINITY, l = 0.f;
      bool ok = true;
      for (int i = 0; i < SPI; ++i, ++g) {
        if (!wwait(s_full, (uint32_t)(g & 1))) { ok = false; break; }
        tc05::fence_after();
        if (!busy && lane == 0)  // nothing to read: S is free at once
          asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(s_free) : "memory");
        const int bad = (int)(~page_ok >> (4 * i)) & 0xF;  // 16-token groups whose page is out of range
        float alpha = 1.f, ref = 0.f;
        if (busy) {
          // Pass 1: the step's maximum, 32 columns at a time.
          float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t sr[32];
            tc05::ld32(row_t + S::kSCol + 32 * h, sr);
            tc05::wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const bool okg = !((bad >> (2 * h + (e >> 4))) & 1);
              mx4[e & 3] = fmaxf(mx4[e & 3], okg ? __uint_as_float(sr[e]) * a.qk_scale_log2 : -INFINITY);
            }
          }
          const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
          if (mx > m_use + 8.f) {
            alpha = m_use == -INFINITY ? 0.f : ex2_approx(m_use - mx);
            m_use = mx;
          }
          ref = m_use == -INFINITY ? 0.f : m_use;
        }
        // O is rescaled before this step's P . V is added (MMA2 of step g waits for p_full(g)).
        if (busy && i > 0 && __any_sync(kFull, alpha != 1.f)) {
          if (!wwait(o_done((int)((g - 1) & 1)), (uint32_t)(((g - 1) >> 1) & 1))) { ok = false; break; }
          tc05::fence_after();
#pragma unroll 1
          for (int cb = 0; cb < D / 16; ++cb) {
            uint32_t ov[16];
            tc05::ld16(row_t + S::kOCol + 16 * cb, ov);
            tc05::wait_ld();
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) ov[jj] = __float_as_uint(__uint_as_float(ov[jj]) * alpha);
            tc05::st16(row_t + S::kOCol + 16 * cb, ov);
          }
        }
        // P buffer g & 1 was last read by O += P.V of step g - 2.
        if (g >= 2 && !wwait(o_done((int)(g & 1)), (uint32_t)(((g - 2) >> 1) & 1))) { ok = false; break; }
        tc05::fence_after();
        // Pass 2: weights, 32 columns at a time, stored as 16-bit pairs.
        if (busy) {
          float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t sr[32];
            tc05::ld32(row_t + S::kSCol + 32 * h, sr);
            tc05::wait_ld();
            if (h == 1) {  // S has been read out: the next S may be computed
              tc05::fence_before();
              __syncwarp();
              if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(s_free) : "memory");
            }
            uint32_t pk[16];
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
              const int e0 = 2 * jj, e1 = 2 * jj + 1;
              const bool okg = !((bad >> (2 * h + (e0 >> 4))) & 1);
              const float p0 = okg ? ex2_approx(__uint_as_float(sr[e0]) * a.qk_scale_log2 - ref) : 0.f;
              const float p1 = okg ? ex2_approx(__uint_as_float(sr[e1]) * a.qk_scale_log2 - ref) : 0.f;
              ls[jj & 3] += p0 + p1;
              pk[jj] = pack2<T>(p0, p1);
            }
            tc05::st16(row_t + S::kPCol + 32 * (uint32_t)(g & 1) + 16 * h, pk);
          }
          l = l * alpha + ((ls[0] + ls[1]) + (ls[2] + ls[3]));
          tc05::wait_st();
        }
        // P of step g is in TMEM.
        tc05::fence_before();
        __syncwarp();
        if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(p_full((int)(g & 1))) : "memory");
      }
      if (!ok) break;
      // Epilogue: the item's last O += P.V (step g - 1) has to complete.
      const int64_t gl = g - 1;
      if (!wwait(o_done((int)(gl & 1)), (uint32_t)((gl >> 1) & 1))) break;
      tc05::fence_after();
      if (busy) {
        const int32_t prow = prow_s[tid];
        const float inv = l > 0.f ? 1.f / l : 0.f;
        constexpr int kTileStride = 20;  // floats; 16-byte accesses conflict-free both ways
        float* tile = reinterpret_cast<float*>(base_ptr + S::kQOff) + warp * 32 * kTileStride;
        float4* wr = reinterpret_cast<float4*>(tile + lane * kTileStride);
        const int rsub = lane >> 2, csub = lane & 3;
#pragma unroll 1
        for (int cb = 0; cb < D / 16; ++cb) {
          uint32_t ov[16];
          tc05::ld16(row_t + S::kOCol + 16 * cb, ov);
          tc05::wait_ld();
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4)
            wr[q4] = make_float4(__uint_as_float(ov[4 * q4]) * inv, __uint_as_float(ov[4 * q4 + 1]) * inv,
                                 __uint_as_float(ov[4 * q4 + 2]) * inv, __uint_as_float(ov[4 * q4 + 3]) * inv);
          __syncwarp();
          float4 v[4];
          int32_t pr[4];
#pragma unroll
          for (int ii = 0; ii < 4; ++ii) {
            pr[ii] = __shfl_sync(kFull, prow, 8 * ii + rsub);
            v[ii] = *reinterpret_cast<const float4*>(tile + (8 * ii + rsub) * kTileStride + 4 * csub);
          }
          __syncwarp();
#pragma unroll
          for (int ii = 0; ii < 4; ++ii)
            if (pr[ii] >= 0) *reinterpret_cast<float4*>(a.o_part + (int64_t)pr[ii] * D + 16 * cb + 4 * csub) = v[ii];
        }
        if (prow >= 0) {
          a.m_part[prow] = m_use == -INFINITY ? -INFINITY : m_use * kLn2;
          a.l_part[prow] = l;
        }
      }
      tc05::fence_before();
      __syncwarp();
      if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(item_free) : "memory");
    }
  }

  // -- teardown ---------------------------------------------------------------------------------
  __syncthreads();
  if (*abort_flag) {
    if (tid == 0) flag_status(a.status, PA_DEV_TIMEOUT);
    if (warp == 4 && lane == 0)
      for (int64_t gl = prod_g > STAGES ? prod_g - STAGES : 0; gl < prod_g; ++gl) {
        const long long t0 = clock64();
        while (!tc05::mbar_try_wait(kv_full((int)(gl % STAGES)), (uint32_t)((gl / STAGES) & 1)) &&
               clock64() - t0 < kWaitCycles) {
        }
      }
  }
  cp_async_wait<0>();
  tc05::fence_before();
  __syncthreads();
  if (warp == 0) {
    tc05::fence_after();
    tc05::dealloc(tmem, S::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Log-sum-exp merge of the partitions.  A CTA of max(4, WPI) warps serves
// max(4, WPI) / WPI (sequence, query head) items with WPI warps each (WPI
// grows with the partition count).  Warp w of an item merges partitions w,
// w + WPI, ... with its own running maximum (the lanes compute 32 weights per
// round; partial rows are loaded in prefetched groups), then the item's warps
// merge through shared memory the same way.  A partition whose l is 0 adds
// nothing.  Dense form: rows are requested before the weights are known (one
// round trip less).  SPARSE form (the balanced shared-prefix kernel marks slots
// empty, l = 0, without writing their rows, and most slots are such marks):
// the weights first, then only the rows of the slots with a contribution, so
// an unwritten row is never read.  Launched as a programmatic dependent of the kernel that writes the
// partials, it waits for that grid before reading them.
// ---------------------------------------------------------------------------
template <typename T, int D, int WPI, int SPARSE>
__global__ void __launch_bounds__(WPI > 4 ? 32 * WPI : 128) decode_reduce_kernel(const DecodeArgs a, int num_seqs,
                                                                                 const int32_t* list) {
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  constexpr int VPL = D / 32;
  constexpr int NW = WPI > 4 ? WPI : 4;
  constexpr int IPC = NW / WPI;  // items per CTA
  constexpr int UNROLL = VPL <= 4 ? 8 : 4;
  __shared__ float acc_w[NW][D];
  __shared__ float m_w[NW], l_w[NW];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int sub = warp % WPI;  // warp within its item
  // `list` (optional): [0] = count, then the items to merge (the rows whose lane
  // the balanced kernel split); otherwise every (sequence, query head) item.
  const int64_t slot_i = (int64_t)blockIdx.x * IPC + warp / WPI;
  int64_t item = slot_i;
  bool live = item < (int64_t)num_seqs * a.num_q_heads;
  if (list != nullptr) {
    live = slot_i < (int64_t)list[0];
    item = live ? (int64_t)list[1 + slot_i] : 0;
    live = live && item >= 0 && item < (int64_t)num_seqs * a.num_q_heads;
  }
  int np = 0;
  int64_t base = 0;
  if (live) {
    const int b = (int)(item / a.num_q_heads);
    np = (context_of(a, b, false) + kPartition - 1) / kPartition;
    base = item * a.max_partitions;
  }
  bool merge = live && np > 1;

  // This warp's partitions are p = sub + WPI * (lane + 32 c), c = 0, 1, ...
  // Lane `lane` holds m and l of its first one; the first UNROLL partial rows
  // are requested before the max is known, and each group of rows is
  // accumulated while the next group is in flight.
  auto load_rows = [&](float (&x)[UNROLL][VPL], int p0, int k, int cnt) {
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      if (k + u < cnt) {
        const float* src = a.o_part + (base + p0 + WPI * (k + u)) * D + lane * VPL;
        if constexpr (VPL % 4 == 0) {
#pragma unroll
          for (int v = 0; v < VPL / 4; ++v) {
            const float4 f = reinterpret_cast<const float4*>(src)[v];
            x[u][4 * v] = f.x;
            x[u][4 * v + 1] = f.y;
            x[u][4 * v + 2] = f.z;
            x[u][4 * v + 3] = f.w;
          }
        } else {
#pragma unroll
          for (int i = 0; i < VPL; ++i) x[u][i] = src[i];
        }
      } else {
#pragma unroll
        for (int i = 0; i < VPL; ++i) x[u][i] = 0.f;
      }
    }
  };
  const int pf = sub + WPI * lane;
  float m_first = -INFINITY, l_first = 0.f;
  if (merge && pf < np) {
    m_first = a.m_part[base + pf];
    l_first = a.l_part[base + pf];
  }
  if constexpr (SPARSE == 2) {
    // Slot 0 marked done (l = -1): the balanced kernel wrote this row's output
    // (read in the same round trip as the weights).
    if (merge && a.l_part[base] < 0.f) merge = false;
  }
  float x[UNROLL][VPL];
  if constexpr (!SPARSE) load_rows(x, sub, 0, merge ? min(32, (np - sub + WPI - 1) / WPI) : 0);
  float mx = m_first;
  if (merge)
    for (int p = pf + WPI * 32; p < np; p += WPI * 32) mx = fmaxf(mx, a.m_part[base + p]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, off));

  float acc[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) acc[i] = 0.f;
  float lsum = 0.f;
  if (merge && mx != -INFINITY) {
    for (int p0 = sub, c = 0; p0 < np; p0 += WPI * 32, ++c) {
      const int p = p0 + WPI * lane;
      float wt = 0.f, lcur = 0.f;
      if (p < np) {
        const float mp = c == 0 ? m_first : a.m_part[base + p];
        lcur = c == 0 ? l_first : a.l_part[base + p];
        wt = lcur > 0.f ? lcur * expf(mp - mx) : 0.f;
      }
      lsum += wt;
      if constexpr (SPARSE) {
        // Only the slots with a contribution are read, UNROLL rows at a time.
        uint32_t present = __ballot_sync(kFull, wt > 0.f);
        while (present) {
          int idx[UNROLL];
#pragma unroll
          for (int u = 0; u < UNROLL; ++u) {
            idx[u] = present ? __ffs(present) - 1 : -1;
            present &= present - 1;
          }
          float xs[UNROLL][VPL];
#pragma unroll
          for (int u = 0; u < UNROLL; ++u) {
            if (idx[u] >= 0) {
              const float* src = a.o_part + (base + p0 + WPI * idx[u]) * D + lane * VPL;
              if constexpr (VPL % 4 == 0) {
#pragma unroll
                for (int v = 0; v < VPL / 4; ++v) {
                  const float4 f = reinterpret_cast<const float4*>(src)[v];
                  xs[u][4 * v] = f.x;
                  xs[u][4 * v + 1] = f.y;
                  xs[u][4 * v + 2] = f.z;
                  xs[u][4 * v + 3] = f.w;
                }
              } else {
#pragma unroll
                for (int i = 0; i < VPL; ++i) xs[u][i] = src[i];
              }
            }
          }
#pragma unroll
          for (int u = 0; u < UNROLL; ++u) {
            const float wk = __shfl_sync(kFull, wt, idx[u] < 0 ? 0 : idx[u]);
            if (idx[u] >= 0) {
#pragma unroll
              for (int i = 0; i < VPL; ++i) acc[i] = fmaf(wk, xs[u][i], acc[i]);
            }
          }
        }
        continue;
      }
      const int cnt = min(32, (np - p0 + WPI - 1) / WPI);
      if (c > 0) load_rows(x, p0, 0, cnt);
      // One batch of UNROLL rows at a time, the next requested once this one is
      // added (no second buffer: fewer registers, more warps per SM, which is
      // what this latency-bound kernel needs).
      for (int k = 0; k < cnt; k += UNROLL) {
        if (k > 0) load_rows(x, p0, k, cnt);
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
          const float wk = __shfl_sync(kFull, wt, min(k + u, 31));
#pragma unroll
          for (int i = 0; i < VPL; ++i) acc[i] = fmaf(k + u < cnt ? wk : 0.f, x[u][i], acc[i]);
        }
      }
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) lsum += __shfl_xor_sync(kFull, lsum, off);

  if constexpr (WPI == 1) {
    if (merge) {
      T* out = reinterpret_cast<T*>(a.out) + item * D + lane * VPL;
#pragma unroll
      for (int i = 0; i < VPL; ++i) out[i] = from_float<T>(lsum > 0.f ? acc[i] / lsum : 0.f);
    }
  } else {
#pragma unroll
    for (int i = 0; i < VPL; ++i) acc_w[warp][lane * VPL + i] = acc[i];
    if (lane == 0) {
      m_w[warp] = mx;
      l_w[warp] = lsum;
    }
    __syncthreads();
    if (!merge) return;
    const int w0 = warp - sub;  // first warp of this item
    float gm = -INFINITY;
#pragma unroll
    for (int w = 0; w < WPI; ++w) gm = fmaxf(gm, m_w[w0 + w]);
    float scale_w[WPI];
    float total = 0.f;
#pragma unroll
    for (int w = 0; w < WPI; ++w) {
      scale_w[w] = gm == -INFINITY ? 0.f : expf(m_w[w0 + w] - gm);
      total += l_w[w0 + w] * scale_w[w];
    }
    T* out = reinterpret_cast<T*>(a.out) + item * D;
    for (int d = sub * 32 + lane; d < D; d += WPI * 32) {
      float o = 0.f;
#pragma unroll
      for (int w = 0; w < WPI; ++w) o = fmaf(acc_w[w0 + w][d], scale_w[w], o);
      out[d] = from_float<T>(total > 0.f ? o / total : 0.f);
    }
  }
}

// ---------------------------------------------------------------------------
// Several query tokens per sequence (draft verification).  Query token t of T
// sits at position ctx - T + t of its sequence and attends to the keys at or
// before that position.  The rows of a kv head are its (token, query head)
// pairs r = t * G + (h - kvh * G); q, out and the partials are indexed as if
// the sequence had T * H_q query heads (DecodeArgs::num_q_heads holds T * H_q),
// so the log-sum-exp merge kernel serves this path unchanged.
// ---------------------------------------------------------------------------
struct VerifyArgs {
  int num_tokens;    // T
  int q_heads;       // H_q
  int row_groups;    // CTAs per kv head along grid y
  int skip_visible;  // 1: the partitions every token sees in full come from the joint kernel;
                     // 2: every partition of sequences longer than one partition does
};

// Partitions [0, n) of a sequence that all T tokens see in full (none for a
// one-partition sequence, whose row is written without a merge).
__device__ __forceinline__ int verify_visible_partitions(int ctx, int num_tokens) {
  return ctx > kPartition ? max(0, ctx - num_tokens + 1) / kPartition : 0;
}

// Work plan of the joint kernel for a verify call, from the context lengths:
// sequence b's T tokens are T members (ids b * T + t, query rows of T * H_q
// per sequence) reading b's table, in chunks of at most `per_chunk` tokens.
// chunks[b * cps + k] = (b, b * T + k * per_chunk, count, extent); members[i] = i.
// The extent is the partitions every token sees in full (`whole` = 0: the
// per-partition kernels), or the 64-token steps of the whole context for a
// sequence longer than one partition (`whole` = 1: the balanced kernel, which
// applies each row's causal limit).
__global__ void verify_plan_kernel(const DecodeArgs a, int num_seqs, int num_tokens, int per_chunk, int cps,
                                   int whole, int32_t* __restrict__ chunks, int32_t* __restrict__ members,
                                   int32_t* __restrict__ merge_list) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b == 0 && merge_list != nullptr) merge_list[0] = 0;  // the merge's item count
  if (b >= num_seqs) return;
  const int ctx = context_of(a, b, false);
  const int sp = whole ? (ctx > kPartition ? (ctx + 63) / 64 : 0) : verify_visible_partitions(ctx, num_tokens);
  for (int k = 0; k < cps; ++k) {
    const int first = k * per_chunk;
    int4 c;
    c.x = b;
    c.y = b * num_tokens + first;
    c.z = min(per_chunk, num_tokens - first);
    c.w = sp;
    reinterpret_cast<int4*>(chunks)[(int64_t)b * cps + k] = c;
  }
  for (int t = 0; t < num_tokens; ++t) members[(int64_t)b * num_tokens + t] = b * num_tokens + t;
}

// Row of q / out (in units of head_dim) for row r of kv head kvh of sequence b.
__device__ __forceinline__ int64_t verify_row(const DecodeArgs& a, const VerifyArgs& v, int b, int kvh, int r) {
  const int t = r / a.group;
  return (int64_t)b * a.num_q_heads + (int64_t)t * v.q_heads + kvh * a.group + (r - t * a.group);
}

// Number of keys row r sees: positions 0 .. ctx - T + t.
__device__ __forceinline__ int verify_limit(const DecodeArgs& a, const VerifyArgs& v, int ctx, int r) {
  return max(0, ctx - v.num_tokens + 1 + r / a.group);
}

// Final rows, or the partition's partials, of rows [r0, r0 + nr) from the
// per-warp (o, m, l) in shared memory: o_w[w * stride + j * D + d],
// m at ml_w[w * stride + j], l at ml_w[w * stride + rows_cap + j].
template <typename T, int D>
__device__ __forceinline__ void verify_merge_store(const DecodeArgs& a, const VerifyArgs& v, int b, int kvh, int r0,
                                                   int nr, int p, int np, int warps, int stride, int rows_cap,
                                                   const float* o_w, const float* ml_w) {
  for (int i = threadIdx.x; i < nr * D; i += blockDim.x) {
    const int j = i / D;
    const int d = i - j * D;
    float mx = -INFINITY;
    for (int w = 0; w < warps; ++w) mx = fmaxf(mx, ml_w[w * stride + j]);
    float lsum = 0.f, osum = 0.f;
    if (mx != -INFINITY) {
      for (int w = 0; w < warps; ++w) {
        const float c = exp2f(ml_w[w * stride + j] - mx);
        lsum += ml_w[w * stride + rows_cap + j] * c;
        osum += o_w[w * stride + j * D + d] * c;
      }
    }
    const float res = lsum > 0.f ? osum / lsum : 0.f;
    const int64_t row = verify_row(a, v, b, kvh, r0 + j);
    if (np <= 1) {
      reinterpret_cast<T*>(a.out)[row * D + d] = from_float<T>(res);
    } else {
      const int64_t part = row * a.max_partitions + p;
      a.o_part[part * D + d] = res;
      if (d == 0) {
        a.m_part[part] = mx == -INFINITY ? -INFINITY : mx * kLn2;
        a.l_part[part] = lsum;
      }
    }
  }
}

template <typename T, int D>
__device__ __forceinline__ void verify_zero_rows(const DecodeArgs& a, const VerifyArgs& v, int b, int kvh, int r0,
                                                 int nr) {
  for (int i = threadIdx.x; i < nr * D; i += blockDim.x) {
    const int j = i / D;
    reinterpret_cast<T*>(a.out)[verify_row(a, v, b, kvh, r0 + j) * D + (i - j * D)] = from_float<T>(0.f);
  }
}

__device__ __forceinline__ void ldmatrix_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];\n" : "=r"(r0), "=r"(r1) : "r"(addr));
}

// Tensor-core verify kernel.  Grid (num_seqs, num_kv_heads * row_groups, P);
// NW warps stream their runs of 16-token tiles of the partition as in the
// single-query kernel, with 8 * NT query rows (NT n8 MMA tiles) per CTA
// instead of the G heads of one token.  The rows' Q sits in shared memory,
// swizzled like the K/V tiles; a row's causal limit masks the scores of the
// tiles it cuts (the last few tiles of the context), the others run unmasked.
template <int D, int NW, int STAGES, int NT>
struct VerifyShape {
  static constexpr int kRows = 8 * NT;
  static constexpr int kRowBytes = 2 * D;
  static constexpr int kChunksPerRow = kRowBytes / 16;
  static constexpr int kTile = 16;
  static constexpr int kTileBytes = kTile * kRowBytes;
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kMergeBytes = kRows * D * 4 + 2 * kRows * 4;
  static constexpr int kWarpBytes = STAGES * kStageBytes > kMergeBytes ? STAGES * kStageBytes : kMergeBytes;
  static constexpr int kQBytes = kRows * kRowBytes;
  static constexpr int kSmemBytes = kQBytes + NW * kWarpBytes;
  static constexpr int kChunksPerLane = kTile * kChunksPerRow / 32;
};

template <typename T, int D, int NW, int STAGES, int NT>
__global__ void __launch_bounds__(NW * 32) decode_verify_tc_kernel(const DecodeArgs a, const VerifyArgs v) {
  const AfterPrerequisiteGrid after{threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0};
  // The merge, launched after this kernel as a programmatic dependent, may start now (it waits for this grid).
  if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  using S = VerifyShape<D, NW, STAGES, NT>;
  constexpr int KSTEPS = D / 16;
  constexpr int MTILES = D / 16;
  extern __shared__ __align__(128) uint8_t smem[];

  const int b = blockIdx.x;
  const int kvh = blockIdx.y / v.row_groups;
  const int r0 = (blockIdx.y - kvh * v.row_groups) * S::kRows;
  const int nr = min(S::kRows, v.num_tokens * a.group - r0);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2;
  const int t = lane & 3;

  const int ctx = context_of(a, b, threadIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0);
  const int np = (ctx + kPartition - 1) / kPartition;
  // With the joint kernel on the partitions every token sees, grid z counts the ones after them;
  // with the balanced kernel on every sequence longer than one partition, only the others are left.
  const int p = blockIdx.z + (v.skip_visible == 1 ? verify_visible_partitions(ctx, v.num_tokens) : 0);
  if (p >= max(np, 1) || (v.skip_visible == 2 && np > 1)) return;
  if (ctx == 0) {
    verify_zero_rows<T, D>(a, v, b, kvh, r0, nr);
    return;
  }
  const int bs = a.block_size;
  const int tok_begin = p * kPartition;
  const int tok_end = min(ctx, tok_begin + kPartition);
  const int ntiles = (tok_end - tok_begin + S::kTile - 1) / S::kTile;
  const int per_warp = (ntiles + NW - 1) / NW;
  const int first_tile = warp * per_warp;
  const int my_tiles = max(0, min(per_warp, ntiles - first_tile));

  const int first_block = tok_begin / bs;
  const int nblk = (tok_end - 1) / bs - first_block + 1;
  int lane_page = 0;
  if (lane < nblk) lane_page = __ldg(a.block_tables + (int64_t)b * a.max_blocks_per_seq + first_block + lane);

  // Keys each of this lane's score rows (8 nt + 2 t + e) may see; padding rows see none.
  int lim[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int row = 8 * nt + 2 * t + e;
      lim[nt][e] = row < nr ? verify_limit(a, v, ctx, r0 + row) : 0;
    }
  const int lim_min = verify_limit(a, v, ctx, r0);  // smallest limit of a real row here

  const uint32_t q_u32 = smem_u32(smem);
  uint8_t* wsm = smem + S::kQBytes + warp * S::kWarpBytes;
  const uint32_t wsm_u32 = smem_u32(wsm);
  const T* kc = reinterpret_cast<const T*>(a.key_cache);
  const T* vc = reinterpret_cast<const T*>(a.value_cache);

  // The CTA's Q rows (zeros for padding rows): the oldest cp.async group.
  for (int i = threadIdx.x; i < S::kRows * S::kChunksPerRow; i += NW * 32) {
    const int r = i / S::kChunksPerRow;
    const int c = i - r * S::kChunksPerRow;
    const bool ok = r < nr;
    const T* src = reinterpret_cast<const T*>(a.q) + (ok ? verify_row(a, v, b, kvh, r0 + r) : 0) * D + c * 8;
    cp_async_16(q_u32 + r * S::kRowBytes + ((c ^ (r & 7)) << 4), src, ok ? 16u : 0u);
  }
  cp_async_commit();

  auto load_tile = [&](int i, int stage) {
    const int tok0 = tok_begin + (first_tile + i) * S::kTile;
    int valid = min(S::kTile, tok_end - tok0);
    int page = __shfl_sync(kFull, lane_page, tok0 / bs - first_block);
    if ((unsigned)page >= (unsigned)a.num_blocks) {
      if (lane == 0) flag_status(a.status, PA_DEV_BAD_PAGE);
      valid = 0;
      page = 0;
    }
    const int64_t row0 = ((int64_t)page * a.num_kv_heads + kvh) * bs + (tok0 % bs);
    const T* ksrc = kc + row0 * D;
    const T* vsrc = vc + row0 * D;
    const uint32_t kdst = wsm_u32 + stage * S::kStageBytes;
    const uint32_t vdst = kdst + S::kTileBytes;
#pragma unroll
    for (int j = 0; j < S::kChunksPerLane; ++j) {
      const int idx = lane + 32 * j;
      const int r = idx / S::kChunksPerRow;
      const int c = idx - r * S::kChunksPerRow;
      const bool ok = r < valid;
      const int64_t src = (int64_t)(ok ? r : 0) * D + c * 8;
      const uint32_t dst = r * S::kRowBytes + ((c ^ (r & 7)) << 4);
      cp_async_16(kdst + dst, ksrc + src, ok ? 16u : 0u);
      cp_async_16(vdst + dst, vsrc + src, ok ? 16u : 0u);
    }
  };

  float o[NT][MTILES][4];
  float m[NT][2], l[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int mt = 0; mt < MTILES; ++mt) o[nt][mt][0] = o[nt][mt][1] = o[nt][mt][2] = o[nt][mt][3] = 0.f;
    m[nt][0] = m[nt][1] = -INFINITY;
    l[nt][0] = l[nt][1] = 0.f;
  }

#pragma unroll
  for (int i = 0; i < STAGES - 1; ++i) {
    if (i < my_tiles) load_tile(i, i);
    cp_async_commit();
  }
  cp_async_wait<STAGES - 1>();  // the Q group
  __syncthreads();

  for (int i = 0; i < my_tiles; ++i) {
    {
      const int nxt = i + STAGES - 1;
      if (nxt < my_tiles) load_tile(nxt, nxt % STAGES);
      cp_async_commit();
    }
    cp_async_wait<STAGES - 1>();
    __syncwarp();

    const int stage = i % STAGES;
    const uint32_t kbase = wsm_u32 + stage * S::kStageBytes;
    const uint32_t vbase = kbase + S::kTileBytes;
    const int tok0 = tok_begin + (first_tile + i) * S::kTile;
    int valid = min(S::kTile, tok_end - tok0);
    {
      const int page = __shfl_sync(kFull, lane_page, tok0 / bs - first_block);
      if ((unsigned)page >= (unsigned)a.num_blocks) valid = 0;
    }

    // S^T = K_tile . Q^T, one n8 tile of rows at a time.
    float s[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
    {
      const int r = (lane & 7) + ((lane >> 3) & 1) * 8;
      const uint32_t rbase = kbase + r * S::kRowBytes;
      const int qr = lane & 7;
#pragma unroll
      for (int ks = 0; ks < KSTEPS; ++ks) {
        const int c = 2 * ks + (lane >> 4);
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4(rbase + ((c ^ (r & 7)) << 4), a0, a1, a2, a3);
        if constexpr (NT == 1) {
          uint32_t b0, b1;
          const int qc = 2 * ks + ((lane >> 3) & 1);
          ldmatrix_x2(q_u32 + qr * S::kRowBytes + ((qc ^ qr) << 4), b0, b1);
          mma_16816<T>(s[0], a0, a1, a2, a3, b0, b1);
        } else {
#pragma unroll
          for (int nt = 0; nt < NT; nt += 2) {
            // Matrices: rows of tile nt (chunks 2ks, 2ks+1), then of tile nt + 1.
            const int qrow = 8 * (nt + (lane >> 4)) + qr;
            const int qc = 2 * ks + ((lane >> 3) & 1);
            uint32_t b0, b1, b2, b3;
            ldmatrix_x4(q_u32 + qrow * S::kRowBytes + ((qc ^ qr) << 4), b0, b1, b2, b3);
            mma_16816<T>(s[nt], a0, a1, a2, a3, b0, b1);
            mma_16816<T>(s[nt + 1], a0, a1, a2, a3, b2, b3);
          }
        }
      }
    }
    // s[nt][0..1]: token g, rows 8 nt + 2t, 2t + 1; s[nt][2..3]: token g + 8.
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[nt][e] *= a.qk_scale_log2;
    if (tok0 + S::kTile > lim_min || valid < S::kTile) {
      const int cut = tok0 + valid;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int lm = min(lim[nt][e], cut);
          if (tok0 + g >= lm) s[nt][e] = -INFINITY;
          if (tok0 + g + 8 >= lm) s[nt][2 + e] = -INFINITY;
        }
    }

    // Each row's reference m (base 2) is raised only when a score passes it by more than 8, so
    // the weights stay below 2^8 and O is rescaled rarely; the partials store that reference.
    float tmax[NT][2];
    bool raise = false;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        float mx = fmaxf(s[nt][j], s[nt][2 + j]);
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 16));
        tmax[nt][j] = mx;
        raise |= mx > m[nt][j] + 8.f;
      }
    if (__any_sync(kFull, raise)) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        float alpha[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const float mn = fmaxf(m[nt][j], tmax[nt][j]);
          alpha[j] = ex2_approx(m[nt][j] - (mn == -INFINITY ? 0.f : mn));
          l[nt][j] *= alpha[j];
          m[nt][j] = mn;
        }
#pragma unroll
        for (int mt = 0; mt < MTILES; ++mt) {
          o[nt][mt][0] *= alpha[0];
          o[nt][mt][1] *= alpha[1];
          o[nt][mt][2] *= alpha[0];
          o[nt][mt][3] *= alpha[1];
        }
      }
    }

    uint32_t pb[NT][2], pl[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float pr[4];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const float base = m[nt][j] == -INFINITY ? 0.f : m[nt][j];
        pr[j] = ex2_approx(s[nt][j] - base);
        pr[2 + j] = ex2_approx(s[nt][2 + j] - base);
        l[nt][j] += pr[j] + pr[2 + j];
      }
      // P^T as the B operand, a 16-bit high part plus the rounding residual.
      const uint32_t hi0 = pack2<T>(pr[0], pr[1]);
      const uint32_t hi1 = pack2<T>(pr[2], pr[3]);
      const float2 q0 = unpack2<T>(hi0), q1 = unpack2<T>(hi1);
      pb[nt][0] = movmatrix_trans(hi0);
      pb[nt][1] = movmatrix_trans(hi1);
      pl[nt][0] = movmatrix_trans(pack2<T>(pr[0] - q0.x, pr[1] - q0.y));
      pl[nt][1] = movmatrix_trans(pack2<T>(pr[2] - q1.x, pr[3] - q1.y));
    }

    // O^T += V_tile^T . P^T for every row tile, one m16 tile of head_dim at a time.
    {
      const int mat = lane >> 3;
      const int r = (lane & 7) + ((mat >> 1) << 3);
      const uint32_t rbase = vbase + r * S::kRowBytes;
#pragma unroll
      for (int mt = 0; mt < MTILES; ++mt) {
        const int c = 2 * mt + (mat & 1);
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4_trans(rbase + ((c ^ (r & 7)) << 4), a0, a1, a2, a3);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          mma_16816<T>(o[nt][mt], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
          mma_16816<T>(o[nt][mt], a0, a1, a2, a3, pl[nt][0], pl[nt][1]);
        }
      }
    }
    __syncwarp();
  }
  cp_async_wait<0>();
  __syncwarp();

  // Warp partials into this warp's region: o[kRows][D], then m[kRows], l[kRows].
  float* o_w = reinterpret_cast<float*>(wsm);
  float* ml_w = o_w + S::kRows * D;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      l[nt][j] += __shfl_xor_sync(kFull, l[nt][j], 4);
      l[nt][j] += __shfl_xor_sync(kFull, l[nt][j], 8);
      l[nt][j] += __shfl_xor_sync(kFull, l[nt][j], 16);
    }
    const int rr = 8 * nt + 2 * t;
#pragma unroll
    for (int mt = 0; mt < MTILES; ++mt) {
      const int d = 16 * mt + g;
      o_w[rr * D + d] = o[nt][mt][0];
      o_w[(rr + 1) * D + d] = o[nt][mt][1];
      o_w[rr * D + d + 8] = o[nt][mt][2];
      o_w[(rr + 1) * D + d + 8] = o[nt][mt][3];
    }
    if (g == 0) {
      ml_w[rr] = m[nt][0];
      ml_w[rr + 1] = m[nt][1];
      ml_w[S::kRows + rr] = l[nt][0];
      ml_w[S::kRows + rr + 1] = l[nt][1];
    }
  }
  __syncthreads();
  const float* base_f = reinterpret_cast<const float*>(smem + S::kQBytes);
  verify_merge_store<T, D>(a, v, b, kvh, r0, nr, p, np, NW, S::kWarpBytes / 4, S::kRows, base_f,
                           base_f + S::kRows * D);
}

// CUDA-core verify kernel (fp32, or block sizes off the 16-token tile).
// Grid (num_seqs, num_kv_heads * row_groups, P); a CTA serves GC rows.
template <typename T, int D, int GC, int NW>
__global__ void __launch_bounds__(NW * 32) decode_verify_cc_kernel(const DecodeArgs a, const VerifyArgs v) {
  constexpr int VPL = D / 32;
  constexpr int kStride = GC * D + 2 * GC;
  __shared__ float w_s[NW * kStride];

  const int b = blockIdx.x;
  const int kvh = blockIdx.y / v.row_groups;
  const int r0 = (blockIdx.y - kvh * v.row_groups) * GC;
  const int nr = min(GC, v.num_tokens * a.group - r0);
  const int p = blockIdx.z;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int ctx = context_of(a, b, threadIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0);
  const int np = (ctx + kPartition - 1) / kPartition;
  if (p >= max(np, 1)) return;
  if (ctx == 0) {
    verify_zero_rows<T, D>(a, v, b, kvh, r0, nr);
    return;
  }
  const int tok_begin = p * kPartition;
  const int tok_end = min(ctx, tok_begin + kPartition);

  float qv[GC][VPL];
  int lim[GC];
#pragma unroll
  for (int j = 0; j < GC; ++j) {
    lim[j] = j < nr ? verify_limit(a, v, ctx, r0 + j) : 0;
    if (j < nr) {
      load_floats<T, VPL>(reinterpret_cast<const T*>(a.q) + verify_row(a, v, b, kvh, r0 + j) * D + lane * VPL,
                          qv[j]);
#pragma unroll
      for (int i = 0; i < VPL; ++i) qv[j][i] *= a.qk_scale_log2;
    } else {
#pragma unroll
      for (int i = 0; i < VPL; ++i) qv[j][i] = 0.f;
    }
  }
  float m[GC], l[GC], o[GC][VPL];
#pragma unroll
  for (int j = 0; j < GC; ++j) {
    m[j] = -INFINITY;
    l[j] = 0.f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) o[j][i] = 0.f;
  }

  const T* kc = reinterpret_cast<const T*>(a.key_cache);
  const T* vc = reinterpret_cast<const T*>(a.value_cache);
  const int32_t* table = a.block_tables + (int64_t)b * a.max_blocks_per_seq;
  for (int tok = tok_begin + warp; tok < tok_end; tok += NW) {
    const int page = __ldg(table + tok / a.block_size);
    if ((unsigned)page >= (unsigned)a.num_blocks) {
      if (lane == 0) flag_status(a.status, PA_DEV_BAD_PAGE);
      continue;
    }
    const int64_t row =
        (((int64_t)page * a.num_kv_heads + kvh) * a.block_size + tok % a.block_size) * D + lane * VPL;
    float kf[VPL], vf[VPL];
    load_floats<T, VPL>(kc + row, kf);
    load_floats<T, VPL>(vc + row, vf);
    float s[GC];
#pragma unroll
    for (int j = 0; j < GC; ++j) {
      float acc = 0.f;
#pragma unroll
      for (int i = 0; i < VPL; ++i) acc = fmaf(qv[j][i], kf[i], acc);
      s[j] = acc;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
#pragma unroll
      for (int j = 0; j < GC; ++j) s[j] += __shfl_xor_sync(kFull, s[j], off);
    }
#pragma unroll
    for (int j = 0; j < GC; ++j) {
      if (tok >= lim[j]) continue;  // after this row's position (uniform across the warp)
      const float mn = fmaxf(m[j], s[j]);
      const float alpha = exp2f(m[j] - mn);
      const float pr = exp2f(s[j] - mn);
      l[j] = l[j] * alpha + pr;
#pragma unroll
      for (int i = 0; i < VPL; ++i) o[j][i] = fmaf(pr, vf[i], o[j][i] * alpha);
      m[j] = mn;
    }
  }

  float* mine = w_s + warp * kStride;
#pragma unroll
  for (int j = 0; j < GC; ++j) {
#pragma unroll
    for (int i = 0; i < VPL; ++i) mine[j * D + lane * VPL + i] = o[j][i];
    if (lane == 0) {
      mine[GC * D + j] = m[j];
      mine[GC * D + GC + j] = l[j];
    }
  }
  __syncthreads();
  verify_merge_store<T, D>(a, v, b, kvh, r0, nr, p, np, NW, kStride, GC, w_s, w_s + GC * D);
}

// ---------------------------------------------------------------------------
// Host side.
// ---------------------------------------------------------------------------
std::atomic<int> g_kernel_choice{PA_DECODE_AUTO};
std::atomic<int> g_fault{PA_FAULT_NONE};
std::atomic<int> g_tc_warps{4};
std::atomic<int> g_tc_stages{2};
std::atomic<int> g_verify_rows{0};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct WorkspaceLayout {
  size_t o_off, m_off, l_off, total;
};

WorkspaceLayout workspace_layout(int64_t num_seqs, int64_t num_q_heads, int64_t head_dim, int64_t partitions) {
  const size_t rows = (size_t)num_seqs * num_q_heads * partitions;
  WorkspaceLayout w;
  w.o_off = 0;
  w.m_off = align256(rows * head_dim * sizeof(float));
  w.l_off = w.m_off + align256(rows * sizeof(float));
  w.total = w.l_off + align256(rows * sizeof(float));
  return w;
}

// Sets the kernel's dynamic shared-memory limit once per device.
template <typename Kernel>
cudaError_t ensure_smem(Kernel kernel, int bytes, std::atomic<uint64_t>& done) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  const uint64_t bit = dev < 64 ? (1ull << dev) : 0;
  if (bit && (done.load() & bit)) return cudaSuccess;
  err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (err == cudaSuccess && bit) done.fetch_or(bit);
  return err;
}

template <typename T, int D, int NW, int STAGES>
cudaError_t launch_tc(const DecodeArgs& a, dim3 grid, cudaStream_t stream, bool dependent) {
  using S = TcShape<D, NW, STAGES>;
  static std::atomic<uint64_t> done{0};
  auto kernel = decode_tc_kernel<T, D, NW, STAGES>;
  cudaError_t err = ensure_smem(kernel, S::kSmemBytes, done);
  if (err != cudaSuccess) return err;
  if (!dependent) {
    kernel<<<grid, NW * 32, S::kSmemBytes, stream>>>(a);
    return cudaGetLastError();
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(NW * 32);
  cfg.dynamicSmemBytes = S::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, a);
}

template <typename T, int D>
cudaError_t launch_tc_config(const DecodeArgs& a, dim3 grid, cudaStream_t stream, int warps, int stages,
                             bool dependent) {
  if (warps == 4 && stages == 3) return launch_tc<T, D, 4, 3>(a, grid, stream, dependent);
  if (warps == 4 && stages == 2) return launch_tc<T, D, 4, 2>(a, grid, stream, dependent);
  if (warps == 4 && stages == 4) return launch_tc<T, D, 4, 4>(a, grid, stream, dependent);
  if (warps == 2 && stages == 4) return launch_tc<T, D, 2, 4>(a, grid, stream, dependent);
  if (warps == 8 && stages == 2) return launch_tc<T, D, 8, 2>(a, grid, stream, dependent);
  return cudaErrorInvalidValue;
}

template <typename T>
cudaError_t launch_tc_dim(const DecodeArgs& a, int head_dim, dim3 grid, cudaStream_t stream, int warps,
                          int stages, bool dependent = false) {
  switch (head_dim) {
    case 64: return launch_tc_config<T, 64>(a, grid, stream, warps, stages, dependent);
    case 128: return launch_tc_config<T, 128>(a, grid, stream, warps, stages, dependent);
    case 256:
      // 256-wide rows: keep to configurations within the shared-memory limit.
      if (warps * stages * 16384 > 200 * 1024) return cudaErrorInvalidValue;
      return launch_tc_config<T, 256>(a, grid, stream, warps, stages, dependent);
  }
  return cudaErrorInvalidValue;
}

template <typename T, int D>
cudaError_t launch_shared(const DecodeArgs& a, dim3 grid, const int32_t* chunks, const int32_t* members,
                          int num_members, int num_seqs, cudaStream_t stream) {
  constexpr int kStages = 4;
  using S = SharedShape<D, kStages>;
  static std::atomic<uint64_t> done{0};
  // Shared partitions are always whole 512-token partitions, where the 16-bit
  // rounding of P averages out; the per-sequence kernel keeps the residual
  // for short and ragged partitions.
  auto kernel = decode_shared_kernel<T, D, kStages, false>;
  cudaError_t err = ensure_smem(kernel, S::kSmemBytes, done);
  if (err != cudaSuccess) return err;
  kernel<<<grid, S::kThreads, S::kSmemBytes, stream>>>(a, chunks, members, num_members, num_seqs);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_shared_tc05(const DecodeArgs& a, dim3 grid, const int32_t* chunks, const int32_t* members,
                               int num_members, int num_seqs, cudaStream_t stream) {
  using S = Tc05Shape<D>;
  static std::atomic<uint64_t> done{0};
  auto kernel = decode_shared_tc05_kernel<T, D>;
  cudaError_t err = ensure_smem(kernel, S::kSmemBytes, done);
  if (err != cudaSuccess) return err;
  kernel<<<grid, S::kThreads, S::kSmemBytes, stream>>>(a, chunks, members, num_members, num_seqs);
  return cudaGetLastError();
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static std::atomic<PFN_cuTensorMapEncodeTiled_v12000> fn{nullptr};
  PFN_cuTensorMapEncodeTiled_v12000 f = fn.load();
  if (!f) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess && ptr) {
      f = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
      fn.store(f);
    }
  }
  return f;
}

// 2-D map of a cache viewed as [num_blocks * num_kv_heads * block_size rows][head_dim],
// boxes of 16 rows x 64 elements (one 128-byte-swizzle block of 16 tokens).
bool encode_cache_map(CUtensorMap* map, const void* cache, pa_dtype dtype, int64_t rows, int head_dim) {
  PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
  if (!encode) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)head_dim, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)head_dim * 2};
  const cuuint32_t box[2] = {64, 16};
  const cuuint32_t elem[2] = {1, 1};
  return encode(map, dtype == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                const_cast<void*>(cache), dims, strides, box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE,
                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
  static std::atomic<int> cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  int n = cached[dev].load();
  if (n <= 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev].store(n);
  }
  return n;
}

template <typename T, int D>
cudaError_t launch_shared_tc05p(const DecodeArgs& a, const CUtensorMap& mk, const CUtensorMap& mv, int num_chunks,
                                const int32_t* chunks, const int32_t* members, int num_members, int num_seqs,
                                int max_sp, cudaStream_t stream) {
  // As many ring stages as shared memory holds: a stage stays with the
  // consumer for about two steps, the rest are loads in flight.
  constexpr int kStages = D == 128 ? 5 : 8;
  using S = Tc05pShape<D, kStages>;
  static std::atomic<uint64_t> done{0};
  auto kernel = decode_shared_tc05p_kernel<T, D, kStages>;
  cudaError_t err = ensure_smem(kernel, S::kSmemBytes, done);
  if (err != cudaSuccess) return err;
  const int64_t items = (int64_t)max_sp * a.num_kv_heads * num_chunks;
  const int grid = (int)(items < sm_count() ? items : sm_count());
  kernel<<<grid, S::kThreads, S::kSmemBytes, stream>>>(a, mk, mv, chunks, num_chunks, members, num_members, num_seqs,
                                                       max_sp, g_fault.load());
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_shared_tc05d(const DecodeArgs& a, const CUtensorMap& mk, const CUtensorMap& mv, int num_chunks,
                                const int32_t* chunks, const int32_t* members, int num_members, int num_seqs,
                                int max_sp, cudaStream_t stream) {
  constexpr int kStages = D == 128 ? 2 : 4;
  using S = Tc05dShape<D, kStages>;
  static std::atomic<uint64_t> done{0};
  auto kernel = decode_shared_tc05d_kernel<T, D, kStages>;
  cudaError_t err = ensure_smem(kernel, S::kSmemBytes, done);
  if (err != cudaSuccess) return err;
  // Two CTAs per SM need the largest shared-memory carveout.
  static std::atomic<uint64_t> carve{0};
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess && dev < 64 && !(carve.load() & (1ull << dev))) {
    err = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (err != cudaSuccess) return err;
    carve.fetch_or(1ull << dev);
  }
  const int64_t items = (int64_t)max_sp * a.num_kv_heads * num_chunks;
  const int64_t slots = 2 * (int64_t)sm_count();
  const int grid = (int)(items < slots ? items : slots);
  kernel<<<grid, S::kThreads, S::kSmemBytes, stream>>>(a, mk, mv, chunks, num_chunks, members, num_members, num_seqs,
                                                       max_sp, g_fault.load());
  return cudaGetLastError();
}

// The balanced tcgen05 kernel: one CTA per SM (CTAs past the work's last range
// exit at once).  `dependent`: a per-sequence kernel runs before it on the stream.
template <typename T, int D>
cudaError_t launch_shared_seg(const DecodeArgs& a, pa_dtype dtype, int num_chunks, const int32_t* chunks,
                              const int32_t* members, int num_members, const int32_t* first_partition, int num_seqs,
                              bool dependent, cudaStream_t stream, bool fold_tails = true, int verify_tokens = 0,
                              int32_t* merge_list = nullptr) {
  constexpr int kStages = D == 128 ? 5 : 8;
  using S = SegShape<D, kStages>;
  static std::atomic<uint64_t> done[2] = {{0}, {0}};
  auto kernel = verify_tokens > 0 ? decode_shared_seg_kernel<T, D, kStages, true>
                                  : decode_shared_seg_kernel<T, D, kStages, false>;
  cudaError_t err = ensure_smem(kernel, S::kSmemBytes, done[verify_tokens > 0 ? 1 : 0]);
  if (err != cudaSuccess) return err;
  // K and V go through the tensor-memory-access unit when the caches fit tensor
  // maps (cp.async otherwise, and for V groups the context ends inside).
  CUtensorMap mk, mv;
  std::memset(&mk, 0, sizeof(mk));
  std::memset(&mv, 0, sizeof(mv));
  const int64_t rows = (int64_t)a.num_blocks * a.num_kv_heads * a.block_size;
  const int tma_k = rows < (1ll << 31) && encode_cache_map(&mk, a.key_cache, dtype, rows, D) &&
                            encode_cache_map(&mv, a.value_cache, dtype, rows, D)
                        ? 1
                        : 0;
  // Always a programmatic dependent: after a per-sequence kernel (`dependent`) it
  // reads inputs that kernel does not write and only waits for it at the end; after
  // any other kernel it waits before its first read.
  return launch_pdl(kernel, dim3(sm_count()), dim3(S::kThreads), S::kSmemBytes, stream, true, a, mk, mv, tma_k,
                    chunks, num_chunks, members, num_members, first_partition, num_seqs, fold_tails ? 1 : 0,
                    verify_tokens, dependent ? 0 : 1, (int)g_fault.load(), merge_list);
}

std::atomic<int> g_shared_kernel{PA_SHARED_PREFIX_AUTO};

template <typename T>
cudaError_t launch_shared_dim(const DecodeArgs& a, int head_dim, dim3 grid, const int32_t* chunks,
                              const int32_t* members, int num_members, int num_seqs, pa_dtype dtype,
                              cudaStream_t stream) {
  const int choice = g_shared_kernel.load();
  if (choice == PA_SHARED_PREFIX_AUTO || choice == PA_SHARED_PREFIX_TCGEN05 ||
      choice == PA_SHARED_PREFIX_TCGEN05_2CTA || choice == PA_SHARED_PREFIX_TCGEN05_ITEMS) {
    const int64_t rows = (int64_t)a.num_blocks * a.num_kv_heads * a.block_size;
    CUtensorMap mk, mv;
    if (rows < (1ll << 31) && encode_cache_map(&mk, a.key_cache, dtype, rows, head_dim) &&
        encode_cache_map(&mv, a.value_cache, dtype, rows, head_dim)) {
      const bool two = choice == PA_SHARED_PREFIX_TCGEN05_2CTA;
      if (head_dim == 64)
        return two ? launch_shared_tc05d<T, 64>(a, mk, mv, grid.x, chunks, members, num_members, num_seqs, grid.z,
                                                stream)
                   : launch_shared_tc05p<T, 64>(a, mk, mv, grid.x, chunks, members, num_members, num_seqs, grid.z,
                                                stream);
      if (head_dim == 128)
        return two ? launch_shared_tc05d<T, 128>(a, mk, mv, grid.x, chunks, members, num_members, num_seqs, grid.z,
                                                 stream)
                   : launch_shared_tc05p<T, 128>(a, mk, mv, grid.x, chunks, members, num_members, num_seqs, grid.z,
                                                 stream);
    }
  }
  const bool tc05 = choice != PA_SHARED_PREFIX_MMA_SYNC;
  switch (head_dim) {
    case 64:
      return tc05 ? launch_shared_tc05<T, 64>(a, grid, chunks, members, num_members, num_seqs, stream)
                  : launch_shared<T, 64>(a, grid, chunks, members, num_members, num_seqs, stream);
    case 128:
      return tc05 ? launch_shared_tc05<T, 128>(a, grid, chunks, members, num_members, num_seqs, stream)
                  : launch_shared<T, 128>(a, grid, chunks, members, num_members, num_seqs, stream);
  }
  return cudaErrorInvalidValue;
}

constexpr int kCcHeads = 4;
constexpr int kCcWarps = 4;

template <typename T>
cudaError_t launch_cc(const DecodeArgs& a, int head_dim, int num_seqs, int partitions, cudaStream_t stream) {
  const int chunks = (a.group + kCcHeads - 1) / kCcHeads;
  dim3 grid(num_seqs, a.num_kv_heads * chunks, partitions - a.partition_base);
  switch (head_dim) {
    case 64: decode_cc_kernel<T, 64, kCcHeads, kCcWarps><<<grid, kCcWarps * 32, 0, stream>>>(a); break;
    case 128: decode_cc_kernel<T, 128, kCcHeads, kCcWarps><<<grid, kCcWarps * 32, 0, stream>>>(a); break;
    case 256: decode_cc_kernel<T, 256, kCcHeads, kCcWarps><<<grid, kCcWarps * 32, 0, stream>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

// Launch with programmatic stream serialisation when `dependent` (the kernel
// may start before the one before it on the stream finishes, and waits for it
// with griddepcontrol.wait), as an ordinary launch otherwise.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       bool dependent, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = dependent ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

template <typename T, int D, int SPARSE>
cudaError_t launch_reduce_dim(const DecodeArgs& a, int num_seqs, cudaStream_t stream, bool dependent,
                              const int32_t* list, int64_t list_cap) {
  const int64_t items = list ? std::min<int64_t>(list_cap, (int64_t)num_seqs * a.num_q_heads)
                             : (int64_t)num_seqs * a.num_q_heads;
  auto grid = [&](int ipc) { return dim3((unsigned)((items + ipc - 1) / ipc)); };
  // Warps per (sequence, query head), by partition count (an 8-warp form,
  // tried for more than 32 partitions, measured no faster).
  if (a.max_partitions <= 16)
    return launch_pdl(decode_reduce_kernel<T, D, 1, SPARSE>, grid(4), dim3(128), 0, stream, dependent, a, num_seqs,
                      list);
  if (a.max_partitions <= 48)
    return launch_pdl(decode_reduce_kernel<T, D, 2, SPARSE>, grid(2), dim3(128), 0, stream, dependent, a, num_seqs,
                      list);
  return launch_pdl(decode_reduce_kernel<T, D, 4, SPARSE>, grid(1), dim3(128), 0, stream, dependent, a, num_seqs,
                    list);
}

template <typename T>
cudaError_t launch_reduce(const DecodeArgs& a, int head_dim, int num_seqs, cudaStream_t stream,
                          bool dependent = false, int sparse = 0, const int32_t* list = nullptr,
                          int64_t list_cap = 0) {
  if ((int64_t)num_seqs * a.num_q_heads > 0x7fffffffLL) return cudaErrorInvalidValue;
  // sparse: 0 every slot written; 1 empty slots marked l = 0; 2 also rows marked done
  auto pick = [&](auto d) -> cudaError_t {
    constexpr int Dv = decltype(d)::value;
    if (sparse == 2) return launch_reduce_dim<T, Dv, 2>(a, num_seqs, stream, dependent, list, list_cap);
    if (sparse == 1) return launch_reduce_dim<T, Dv, 1>(a, num_seqs, stream, dependent, list, list_cap);
    return launch_reduce_dim<T, Dv, 0>(a, num_seqs, stream, dependent, list, list_cap);
  };
  switch (head_dim) {
    case 64: return pick(std::integral_constant<int, 64>{});
    case 128: return pick(std::integral_constant<int, 128>{});
    case 256: return pick(std::integral_constant<int, 256>{});
  }
  return cudaErrorInvalidValue;
}

// `v.skip_visible`: launched as a programmatic dependent of the joint kernel,
// which covers the partitions every token sees in full (1) or every partition
// of the sequences longer than one (2).
template <typename T, int D, int NW, int STAGES, int NT>
cudaError_t launch_verify_tc(const DecodeArgs& a, VerifyArgs v, int num_seqs, int partitions, cudaStream_t stream) {
  using S = VerifyShape<D, NW, STAGES, NT>;
  static std::atomic<uint64_t> done{0};
  auto kernel = decode_verify_tc_kernel<T, D, NW, STAGES, NT>;
  cudaError_t err = ensure_smem(kernel, S::kSmemBytes, done);
  if (err != cudaSuccess) return err;
  v.row_groups = (v.num_tokens * a.group + S::kRows - 1) / S::kRows;
  if ((int64_t)a.num_kv_heads * v.row_groups > 65535) return cudaErrorInvalidValue;
  // After the partitions every token sees a sequence has at most 1 + ceil((T - 1) / 512) left.
  const int tail = 1 + (v.num_tokens - 1 + kPartition - 1) / kPartition;
  const dim3 grid(num_seqs, a.num_kv_heads * v.row_groups,
                  v.skip_visible == 2 ? 1 : v.skip_visible ? std::min(partitions, tail) : partitions);
  if (!v.skip_visible) {
    kernel<<<grid, NW * 32, S::kSmemBytes, stream>>>(a, v);
    return cudaGetLastError();
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(NW * 32);
  cfg.dynamicSmemBytes = S::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, a, v);
}

// Rows per CTA: the fewest n8 tiles that hold a kv head's T * G rows, at most
// 4 (2 at head_dim 256, where the accumulators of more would spill); larger
// row counts take several CTAs per kv head, which read the same pages, mostly
// from L2.
template <typename T, int D>
cudaError_t launch_verify_tc_dim(const DecodeArgs& a, const VerifyArgs& v, int num_seqs, int partitions,
                                 cudaStream_t stream) {
  const int rows = v.num_tokens * a.group;
  // pa_set_verify_tiling may cap the rows per CTA (more row groups, fewer registers per thread).
  const int cap = g_verify_rows.load();
  const int per_cta = std::min(rows <= 8 ? 8 : rows <= 16 ? 16 : 32, cap > 0 ? cap : 32);
  if constexpr (D == 256) {
    if (per_cta <= 8) return launch_verify_tc<T, D, 4, 2, 1>(a, v, num_seqs, partitions, stream);
    return launch_verify_tc<T, D, 4, 2, 2>(a, v, num_seqs, partitions, stream);
  } else {
    if (per_cta <= 8) return launch_verify_tc<T, D, 4, 3, 1>(a, v, num_seqs, partitions, stream);
    if (per_cta <= 16) return launch_verify_tc<T, D, 4, 3, 2>(a, v, num_seqs, partitions, stream);
    return launch_verify_tc<T, D, 4, 3, 4>(a, v, num_seqs, partitions, stream);
  }
}

template <typename T>
cudaError_t launch_verify_cc(const DecodeArgs& a, VerifyArgs v, int head_dim, int num_seqs, int partitions,
                             cudaStream_t stream) {
  v.row_groups = (v.num_tokens * a.group + kCcHeads - 1) / kCcHeads;
  if ((int64_t)a.num_kv_heads * v.row_groups > 65535) return cudaErrorInvalidValue;
  const dim3 grid(num_seqs, a.num_kv_heads * v.row_groups, partitions);
  switch (head_dim) {
    case 64: decode_verify_cc_kernel<T, 64, kCcHeads, kCcWarps><<<grid, kCcWarps * 32, 0, stream>>>(a, v); break;
    case 128: decode_verify_cc_kernel<T, 128, kCcHeads, kCcWarps><<<grid, kCcWarps * 32, 0, stream>>>(a, v); break;
    case 256: decode_verify_cc_kernel<T, 256, kCcHeads, kCcWarps><<<grid, kCcWarps * 32, 0, stream>>>(a, v); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_verify_tc_any(const DecodeArgs& a, const VerifyArgs& v, int head_dim, int num_seqs,
                                 int partitions, cudaStream_t stream) {
  switch (head_dim) {
    case 64: return launch_verify_tc_dim<T, 64>(a, v, num_seqs, partitions, stream);
    case 128: return launch_verify_tc_dim<T, 128>(a, v, num_seqs, partitions, stream);
    case 256: return launch_verify_tc_dim<T, 256>(a, v, num_seqs, partitions, stream);
  }
  return cudaErrorInvalidValue;
}

bool tc_supported(pa_dtype dt, int head_dim, int group, int block_size) {
  return (dt == PA_BF16 || dt == PA_F16) && (head_dim == 64 || head_dim == 128 || head_dim == 256) &&
         group >= 1 && group <= 8 && block_size % 16 == 0 && block_size <= 256;
}

}  // namespace
}  // namespace pa

using namespace pa;

extern "C" pa_status pa_set_decode_kernel(pa_decode_kernel k) {
  if (k != PA_DECODE_AUTO && k != PA_DECODE_CUDA_CORES && k != PA_DECODE_TENSOR_CORES)
    return fail(PA_ERR_INVALID, "pa_set_decode_kernel: unknown kernel %d", (int)k);
  g_kernel_choice.store((int)k);
  return PA_OK;
}

extern "C" pa_status pa_set_fault_injection(int32_t mode) {
  if (mode != PA_FAULT_NONE && mode != PA_FAULT_WITHHOLD_FIRST_ITEM)
    return fail(PA_ERR_INVALID, "pa_set_fault_injection: unknown mode %d", (int)mode);
  g_fault.store(mode);
  return PA_OK;
}

namespace pa {
namespace {
__global__ void eval_exp2_kernel(const float* __restrict__ x, float* __restrict__ y, int64_t n, int method) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    y[i] = method == 0 ? exp2_poly(x[i]) : ex2_approx(x[i]);
}
}  // namespace
}  // namespace pa

extern "C" pa_status pa_eval_exp2(const float* x, float* y, int64_t n, int32_t method, void* stream) {
  if (n < 0 || (n > 0 && (!x || !y)) || (method != 0 && method != 1))
    return fail(PA_ERR_INVALID, "eval_exp2: bad arguments");
  if (n == 0) return PA_OK;
  const int64_t blocks = std::min<int64_t>((n + 255) / 256, 4096);
  eval_exp2_kernel<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n, method);
  const cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return fail(PA_ERR_CUDA, "eval_exp2: %s", cudaGetErrorString(err));
  return PA_OK;
}

extern "C" pa_status pa_set_shared_prefix_kernel(pa_shared_prefix_kernel k) {
  if (k != PA_SHARED_PREFIX_AUTO && k != PA_SHARED_PREFIX_TCGEN05 && k != PA_SHARED_PREFIX_MMA_SYNC &&
      k != PA_SHARED_PREFIX_TCGEN05_SERIAL && k != PA_SHARED_PREFIX_TCGEN05_2CTA &&
      k != PA_SHARED_PREFIX_TCGEN05_ITEMS)
    return fail(PA_ERR_INVALID, "pa_set_shared_prefix_kernel: unknown kernel %d", (int)k);
  g_shared_kernel.store((int)k);
  return PA_OK;
}

extern "C" pa_status pa_set_verify_tiling(int32_t rows_per_cta) {
  if (rows_per_cta != 0 && rows_per_cta != 8 && rows_per_cta != 16 && rows_per_cta != 32)
    return fail(PA_ERR_UNSUPPORTED, "pa_set_verify_tiling: %d rows per CTA (built: 8, 16, 32; 0 = default)",
                rows_per_cta);
  g_verify_rows.store(rows_per_cta);
  return PA_OK;
}

extern "C" pa_status pa_set_decode_tiling(int32_t warps, int32_t stages) {
  const bool ok = (warps == 4 && (stages == 2 || stages == 3 || stages == 4)) || (warps == 2 && stages == 4) ||
                  (warps == 8 && stages == 2);
  if (!ok) return fail(PA_ERR_UNSUPPORTED, "pa_set_decode_tiling: (%d warps, %d stages) not built", warps, stages);
  g_tc_warps.store(warps);
  g_tc_stages.store(stages);
  return PA_OK;
}

extern "C" size_t pa_decode_workspace_size(int32_t num_seqs, int32_t num_q_heads, int32_t head_dim,
                                           int64_t max_context_len) {
  if (num_seqs <= 0 || num_q_heads <= 0 || head_dim <= 0 || max_context_len <= 0) return 0;
  const int64_t partitions = (max_context_len + kPartition - 1) / kPartition;
  if (partitions <= 1) return 0;
  return workspace_layout(num_seqs, num_q_heads, head_dim, partitions).total;
}

namespace {

// Validates a decode call and fills `a`; *partitions receives P.
pa_status prepare_decode(const void* q, const void* key_cache, const void* value_cache, const int32_t* block_tables,
                         int32_t max_blocks_per_seq, const int32_t* context_lens, int32_t num_seqs,
                         int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                         int32_t num_blocks, float scale, void* out, pa_dtype dtype, void* workspace,
                         size_t workspace_bytes, int32_t* dev_status, DecodeArgs& a, int& partitions) {
  if (dtype_bytes(dtype) == 0) return fail(PA_ERR_INVALID, "decode: bad dtype %d", (int)dtype);
  if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0)
    return fail(PA_ERR_INVALID, "decode: num_q_heads must be a positive multiple of num_kv_heads");
  if (head_dim != 64 && head_dim != 128 && head_dim != 256)
    return fail(PA_ERR_UNSUPPORTED, "decode: head_dim %d (supported: 64, 128, 256)", head_dim);
  if (block_size < 1 || block_size > 256) return fail(PA_ERR_UNSUPPORTED, "decode: block_size %d", block_size);
  if (max_blocks_per_seq < 1 || num_blocks < 1) return fail(PA_ERR_INVALID, "decode: empty table or pool");
  if ((int64_t)max_blocks_per_seq * block_size > (1 << 30))
    return fail(PA_ERR_UNSUPPORTED, "decode: max_blocks_per_seq * block_size above 2^30");
  if (num_kv_heads > 65535) return fail(PA_ERR_UNSUPPORTED, "decode: too many kv heads");
  if (!(scale == scale)) return fail(PA_ERR_INVALID, "decode: scale is NaN");
  const int64_t max_ctx = (int64_t)max_blocks_per_seq * block_size;
  partitions = (int)((max_ctx + kPartition - 1) / kPartition);
  if (partitions > 65535) return fail(PA_ERR_UNSUPPORTED, "decode: more than 65535 partitions");
  if (num_seqs == 0) return PA_OK;
  if (!q || !key_cache || !value_cache || !block_tables || !context_lens || !out)
    return fail(PA_ERR_INVALID, "decode: NULL pointer");
  if (!aligned16(q) || !aligned16(key_cache) || !aligned16(value_cache) || !aligned16(out))
    return fail(PA_ERR_INVALID, "decode: q, caches and out must be 16-byte aligned");
  a = DecodeArgs{};
  a.q = q;
  a.key_cache = key_cache;
  a.value_cache = value_cache;
  a.block_tables = block_tables;
  a.context_lens = context_lens;
  a.out = out;
  a.status = dev_status;
  a.max_blocks_per_seq = max_blocks_per_seq;
  a.num_q_heads = num_q_heads;
  a.num_kv_heads = num_kv_heads;
  a.group = num_q_heads / num_kv_heads;
  a.block_size = block_size;
  a.num_blocks = num_blocks;
  a.max_partitions = partitions;
  a.qk_scale_log2 = scale * kLog2e;
  if (partitions > 1) {
    const WorkspaceLayout w = workspace_layout(num_seqs, num_q_heads, head_dim, partitions);
    if (!workspace || workspace_bytes < w.total)
      return fail(PA_ERR_INVALID, "decode: workspace of %zu bytes needed, %zu given", w.total, workspace_bytes);
    if (reinterpret_cast<uintptr_t>(workspace) & 255u)
      return fail(PA_ERR_INVALID, "decode: workspace must be 256-byte aligned");
    char* ws = static_cast<char*>(workspace);
    a.o_part = reinterpret_cast<float*>(ws + w.o_off);
    a.m_part = reinterpret_cast<float*>(ws + w.m_off);
    a.l_part = reinterpret_cast<float*>(ws + w.l_off);
  }
  return PA_OK;
}

// `dependent`: launched as a programmatic dependent of the kernel before it on
// the stream (tensor-core kernel only; the CUDA-core one launches as usual).
pa_status launch_partitions(const DecodeArgs& a, pa_dtype dtype, int head_dim, int num_seqs, int partitions,
                            cudaStream_t s, bool dependent = false) {
  const int choice = g_kernel_choice.load();
  const bool tc_ok = tc_supported(dtype, head_dim, a.group, a.block_size);
  if (choice == PA_DECODE_TENSOR_CORES && !tc_ok)
    return fail(PA_ERR_UNSUPPORTED, "decode: tensor-core kernel needs bf16/f16, G <= 8, block_size %% 16 == 0");
  cudaError_t err;
  if (tc_ok && choice != PA_DECODE_CUDA_CORES) {
    dim3 grid(num_seqs, a.num_kv_heads, partitions - a.partition_base);
    const int warps = g_tc_warps.load(), stages = g_tc_stages.load();
    err = dtype == PA_BF16 ? launch_tc_dim<__nv_bfloat16>(a, head_dim, grid, s, warps, stages, dependent)
                           : launch_tc_dim<__half>(a, head_dim, grid, s, warps, stages, dependent);
  } else {
    err = dtype == PA_F32    ? launch_cc<float>(a, head_dim, num_seqs, partitions, s)
          : dtype == PA_BF16 ? launch_cc<__nv_bfloat16>(a, head_dim, num_seqs, partitions, s)
                             : launch_cc<__half>(a, head_dim, num_seqs, partitions, s);
  }
  if (err != cudaSuccess) return fail(PA_ERR_CUDA, "decode partition kernel: %s", cudaGetErrorString(err));
  return PA_OK;
}

pa_status launch_reduce_any(const DecodeArgs& a, pa_dtype dtype, int head_dim, int num_seqs, cudaStream_t s,
                            bool dependent = false, int sparse = 0, const int32_t* list = nullptr,
                            int64_t list_cap = 0) {
  const cudaError_t err =
      dtype == PA_F32    ? launch_reduce<float>(a, head_dim, num_seqs, s, dependent, sparse, list, list_cap)
      : dtype == PA_BF16 ? launch_reduce<__nv_bfloat16>(a, head_dim, num_seqs, s, dependent, sparse, list, list_cap)
                         : launch_reduce<__half>(a, head_dim, num_seqs, s, dependent, sparse, list, list_cap);
  if (err != cudaSuccess) return fail(PA_ERR_CUDA, "decode reduce kernel: %s", cudaGetErrorString(err));
  return PA_OK;
}

}  // namespace

extern "C" pa_status pa_decode(const void* q, const void* key_cache, const void* value_cache,
                               const int32_t* block_tables, int32_t max_blocks_per_seq,
                               const int32_t* context_lens, int32_t num_seqs, int32_t num_q_heads,
                               int32_t num_kv_heads, int32_t head_dim, int32_t block_size, int32_t num_blocks,
                               float scale, void* out, pa_dtype dtype, void* workspace, size_t workspace_bytes,
                               int32_t* dev_status, void* stream) {
  DecodeArgs a;
  int partitions = 0;
  pa_status st = prepare_decode(q, key_cache, value_cache, block_tables, max_blocks_per_seq, context_lens, num_seqs,
                                num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, scale, out, dtype,
                                workspace, workspace_bytes, dev_status, a, partitions);
  if (st != PA_OK || num_seqs == 0) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // The partition kernel, too, launches as a programmatic dependent of the kernel
  // before it and waits for that grid before its first read.
  a.wait_first = 1;
  st = launch_partitions(a, dtype, head_dim, num_seqs, partitions, s, /*dependent=*/true);
  if (st != PA_OK || partitions <= 1) return st;
  // A programmatic dependent: its CTAs take the SMs the partition kernel's last
  // wave leaves idle and wait there for that grid to finish.
  return launch_reduce_any(a, dtype, head_dim, num_seqs, s, /*dependent=*/true);
}

extern "C" pa_status pa_decode_partitions(const void* q, const void* key_cache, const void* value_cache,
                                          const int32_t* block_tables, int32_t max_blocks_per_seq,
                                          const int32_t* context_lens, int32_t num_seqs, int32_t num_q_heads,
                                          int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                          int32_t num_blocks, float scale, void* out, pa_dtype dtype,
                                          void* workspace, size_t workspace_bytes, int32_t* dev_status,
                                          void* stream) {
  DecodeArgs a;
  int partitions = 0;
  pa_status st = prepare_decode(q, key_cache, value_cache, block_tables, max_blocks_per_seq, context_lens, num_seqs,
                                num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, scale, out, dtype,
                                workspace, workspace_bytes, dev_status, a, partitions);
  if (st != PA_OK || num_seqs == 0) return st;
  a.wait_first = 1;  // a programmatic dependent of the kernel before it (see pa_decode)
  return launch_partitions(a, dtype, head_dim, num_seqs, partitions, static_cast<cudaStream_t>(stream),
                           /*dependent=*/true);
}

extern "C" pa_status pa_decode_reduce(const int32_t* context_lens, int32_t num_seqs, int32_t num_q_heads,
                                      int32_t head_dim, int64_t max_context_len, void* out, pa_dtype dtype,
                                      const void* workspace, size_t workspace_bytes, void* stream) {
  if (dtype_bytes(dtype) == 0) return fail(PA_ERR_INVALID, "decode_reduce: bad dtype %d", (int)dtype);
  if (num_seqs < 0 || num_q_heads <= 0 || max_context_len < 0 || max_context_len > (1 << 30))
    return fail(PA_ERR_INVALID, "decode_reduce: bad sizes");
  if (head_dim != 64 && head_dim != 128 && head_dim != 256)
    return fail(PA_ERR_UNSUPPORTED, "decode_reduce: head_dim %d", head_dim);
  const int partitions = (int)((max_context_len + kPartition - 1) / kPartition);
  if (num_seqs == 0 || partitions <= 1) return PA_OK;
  if (!context_lens || !out) return fail(PA_ERR_INVALID, "decode_reduce: NULL pointer");
  if (!aligned16(out)) return fail(PA_ERR_INVALID, "decode_reduce: out must be 16-byte aligned");
  const WorkspaceLayout w = workspace_layout(num_seqs, num_q_heads, head_dim, partitions);
  if (!workspace || workspace_bytes < w.total)
    return fail(PA_ERR_INVALID, "decode_reduce: workspace of %zu bytes needed, %zu given", w.total, workspace_bytes);
  if (reinterpret_cast<uintptr_t>(workspace) & 255u)
    return fail(PA_ERR_INVALID, "decode_reduce: workspace must be 256-byte aligned");
  DecodeArgs a{};
  a.context_lens = context_lens;
  a.out = out;
  a.num_q_heads = num_q_heads;
  a.max_blocks_per_seq = (int)max_context_len;
  a.block_size = 1;
  a.max_partitions = partitions;
  char* ws = static_cast<char*>(const_cast<void*>(workspace));
  a.o_part = reinterpret_cast<float*>(ws + w.o_off);
  a.m_part = reinterpret_cast<float*>(ws + w.m_off);
  a.l_part = reinterpret_cast<float*>(ws + w.l_off);
  return launch_reduce_any(a, dtype, head_dim, num_seqs, static_cast<cudaStream_t>(stream), /*dependent=*/true);
}

// ---------------------------------------------------------------------------
// pa_decode_verify: T query tokens per sequence, each attending causally.
// ---------------------------------------------------------------------------
namespace {
std::atomic<int> g_verify_path{PA_VERIFY_AUTO};

// Above this many rows (T * G) per kv head AUTO takes the joint path (at 8 rows, one token of a
// group of 8, the per-sequence kernel alone is faster).
constexpr int kVerifyJointRows = 8;

// The partials (the pa_decode layout with T * H_q heads), then the joint kernel's plan:
// chunks int32 [num_seqs * T][4] at most, members int32 [num_seqs * T].
struct VerifyLayout {
  WorkspaceLayout parts;
  size_t chunks_off, members_off, list_off, total;
};

VerifyLayout verify_layout(int64_t num_seqs, int64_t num_tokens, int64_t num_q_heads, int64_t head_dim,
                           int64_t partitions) {
  VerifyLayout v;
  v.parts = workspace_layout(num_seqs, num_tokens * num_q_heads, head_dim, partitions);
  v.chunks_off = v.parts.total;
  v.members_off = v.chunks_off + align256((size_t)num_seqs * num_tokens * 16);
  // the merge's item list: a count, then up to one entry per row
  v.list_off = v.members_off + align256((size_t)num_seqs * num_tokens * 4);
  v.total = v.list_off + align256((1 + (size_t)num_seqs * num_tokens * num_q_heads) * 4);
  return v;
}
}  // namespace

extern "C" pa_status pa_set_verify_path(pa_verify_path path) {
  if (path < PA_VERIFY_AUTO || path > PA_VERIFY_JOINT) return fail(PA_ERR_INVALID, "unknown verify path %d", (int)path);
  g_verify_path.store(path);
  return PA_OK;
}

extern "C" size_t pa_decode_verify_workspace_size(int32_t num_seqs, int32_t num_query_tokens, int32_t num_q_heads,
                                                  int32_t head_dim, int64_t max_context_len) {
  if (num_seqs <= 0 || num_query_tokens <= 0 || num_q_heads <= 0 || head_dim <= 0 || max_context_len <= 0 ||
      (int64_t)num_query_tokens * num_q_heads > (1 << 24))
    return 0;
  const int64_t partitions = (max_context_len + kPartition - 1) / kPartition;
  if (partitions <= 1) return 0;
  return verify_layout(num_seqs, num_query_tokens, num_q_heads, head_dim, partitions).total;
}

extern "C" pa_status pa_decode_verify(const void* q, const void* key_cache, const void* value_cache,
                                      const int32_t* block_tables, int32_t max_blocks_per_seq,
                                      const int32_t* context_lens, int32_t num_seqs, int32_t num_query_tokens,
                                      int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                      int32_t block_size, int32_t num_blocks, float scale, void* out,
                                      pa_dtype dtype, void* workspace, size_t workspace_bytes, int32_t* dev_status,
                                      void* stream) {
  if (num_query_tokens < 1) return fail(PA_ERR_INVALID, "decode_verify: num_query_tokens %d", num_query_tokens);
  if (num_q_heads <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0)
    return fail(PA_ERR_INVALID, "decode_verify: num_q_heads must be a positive multiple of num_kv_heads");
  if ((int64_t)num_query_tokens * num_q_heads > (1 << 24))
    return fail(PA_ERR_UNSUPPORTED, "decode_verify: num_query_tokens * num_q_heads above 2^24");
  // q, out and the partials are laid out as T * H_q query heads per sequence.
  DecodeArgs a;
  int partitions = 0;
  pa_status st = prepare_decode(q, key_cache, value_cache, block_tables, max_blocks_per_seq, context_lens, num_seqs,
                                num_query_tokens * num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                                scale, out, dtype, workspace, workspace_bytes, dev_status, a, partitions);
  if (st != PA_OK || num_seqs == 0) return st;
  const int G = num_q_heads / num_kv_heads;
  a.group = G;
  VerifyArgs v{num_query_tokens, num_q_heads, 0, 0};
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int choice = g_kernel_choice.load();
  const bool tc_ok = (dtype == PA_BF16 || dtype == PA_F16) && block_size % 16 == 0 && block_size <= 256;
  if (choice == PA_DECODE_TENSOR_CORES && !tc_ok)
    return fail(PA_ERR_UNSUPPORTED, "decode_verify: tensor-core kernel needs bf16/f16 and block_size %% 16 == 0");
  cudaError_t err;

  // The partitions all T tokens see in full are a shared prefix of T members:
  // the joint kernel reads each of their pages once for all T * G rows.
  const int path = g_verify_path.load();
  const int per_chunk = G <= PA_PREFIX_QUERIES_PER_CTA ? std::min(num_query_tokens, PA_PREFIX_QUERIES_PER_CTA / G) : 0;
  const int max_visible = (int)std::min<int64_t>((int64_t)max_blocks_per_seq * block_size / kPartition, partitions);
  const bool joint_ok = tc_ok && choice != PA_DECODE_CUDA_CORES && (head_dim == 64 || head_dim == 128) &&
                        partitions > 1 && per_chunk > 0 && max_visible > 0 &&
                        (int64_t)num_seqs * num_query_tokens <= (1 << 26);
  if (path == PA_VERIFY_JOINT && !joint_ok)
    return fail(PA_ERR_UNSUPPORTED, "decode_verify: the joint path needs bf16/f16, head_dim 64 or 128, block_size "
                                    "%% 16 == 0, G <= %d and contexts beyond one partition", PA_PREFIX_QUERIES_PER_CTA);
  const bool joint = joint_ok && (path == PA_VERIFY_JOINT ||
                                  (path == PA_VERIFY_AUTO && (int64_t)num_query_tokens * G > kVerifyJointRows));
  bool balanced = false;  // the balanced joint kernel ran (its merge skips the slots it leaves empty)
  const int32_t* verify_merge_list = nullptr;  // with it: the rows its split lanes left to the merge
  if (joint) {
    const VerifyLayout lay = verify_layout(num_seqs, num_query_tokens, num_q_heads, head_dim, partitions);
    if (workspace_bytes < lay.total)
      return fail(PA_ERR_INVALID, "decode_verify: workspace of %zu bytes needed, %zu given", lay.total,
                  workspace_bytes);
    int32_t* chunks = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + lay.chunks_off);
    int32_t* members = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + lay.members_off);
    int32_t* list = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + lay.list_off);
    verify_merge_list = list;
    const int cps = (num_query_tokens + per_chunk - 1) / per_chunk;
    const int num_members = num_seqs * num_query_tokens;
    // The balanced kernel takes every partition of the sequences longer than one
    // partition, each row up to its own causal limit (its lanes counted in 64-token
    // steps); the per-sequence kernel is left the one-partition sequences.  The
    // per-partition kernels take the partitions every token sees in full.
    const int shared_choice = g_shared_kernel.load();
    const int64_t max_steps = std::min<int64_t>(((int64_t)max_blocks_per_seq * block_size + 63) / 64,
                                                (int64_t)partitions * 8);
    const int64_t units = (int64_t)num_kv_heads * num_seqs * cps * (max_steps + 3);
    balanced = (shared_choice == PA_SHARED_PREFIX_AUTO || shared_choice == PA_SHARED_PREFIX_TCGEN05) &&
               units < kSegMaxUnits;
    verify_plan_kernel<<<(num_seqs + 127) / 128, 128, 0, s>>>(a, num_seqs, num_query_tokens, per_chunk, cps,
                                                                balanced ? 1 : 0, chunks, members,
                                                                balanced ? list : nullptr);
    err = cudaGetLastError();
    if (err != cudaSuccess) return fail(PA_ERR_CUDA, "decode_verify plan kernel: %s", cudaGetErrorString(err));
    // The joint kernel indexes q, the partials and its members with H_q heads per member.
    DecodeArgs aj = a;
    aj.num_q_heads = num_q_heads;
    if (balanced) {
      // It waits for the plan kernel first.  Its members are token ids b * T + t,
      // so they are checked against num_members.
      const int nc = num_seqs * cps;
      const int T = num_query_tokens;
      err = head_dim == 64
                ? (dtype == PA_BF16 ? launch_shared_seg<__nv_bfloat16, 64>(aj, dtype, nc, chunks, members, num_members,
                                                                           nullptr, num_members, false, s, false, T, list)
                                    : launch_shared_seg<__half, 64>(aj, dtype, nc, chunks, members, num_members,
                                                                    nullptr, num_members, false, s, false, T, list))
                : (dtype == PA_BF16 ? launch_shared_seg<__nv_bfloat16, 128>(aj, dtype, nc, chunks, members,
                                                                            num_members, nullptr, num_members, false,
                                                                            s, false, T, list)
                                    : launch_shared_seg<__half, 128>(aj, dtype, nc, chunks, members, num_members,
                                                                     nullptr, num_members, false, s, false, T, list));
    } else {
      const dim3 grid(num_seqs * cps, num_kv_heads, max_visible);
      err = dtype == PA_BF16 ? launch_shared_dim<__nv_bfloat16>(aj, head_dim, grid, chunks, members, num_members,
                                                                num_members, dtype, s)
                             : launch_shared_dim<__half>(aj, head_dim, grid, chunks, members, num_members,
                                                         num_members, dtype, s);
    }
    if (err != cudaSuccess) return fail(PA_ERR_CUDA, "decode_verify joint kernel: %s", cudaGetErrorString(err));
    v.skip_visible = balanced ? 2 : 1;
  }
  if (tc_ok && choice != PA_DECODE_CUDA_CORES)
    err = dtype == PA_BF16 ? launch_verify_tc_any<__nv_bfloat16>(a, v, head_dim, num_seqs, partitions, s)
                           : launch_verify_tc_any<__half>(a, v, head_dim, num_seqs, partitions, s);
  else
    err = dtype == PA_F32    ? launch_verify_cc<float>(a, v, head_dim, num_seqs, partitions, s)
          : dtype == PA_BF16 ? launch_verify_cc<__nv_bfloat16>(a, v, head_dim, num_seqs, partitions, s)
                             : launch_verify_cc<__half>(a, v, head_dim, num_seqs, partitions, s);
  if (err != cudaSuccess) return fail(PA_ERR_CUDA, "decode_verify partition kernel: %s", cudaGetErrorString(err));
  if (partitions <= 1) return PA_OK;
  if (balanced) {
    // Only the rows of the lanes the balanced kernel split need merging: at most
    // one lane of at most PA_PREFIX_QUERIES_PER_CTA rows per CTA boundary.
    const int64_t cap = (int64_t)(sm_count() + 1) * PA_PREFIX_QUERIES_PER_CTA;
    return launch_reduce_any(a, dtype, head_dim, num_seqs, s, /*dependent=*/true, /*sparse=*/2,
                             verify_merge_list, cap);
  }
  return launch_reduce_any(a, dtype, head_dim, num_seqs, s, /*dependent=*/true);
}

// ---------------------------------------------------------------------------
// pa_decode_fixed_scratch: pa_decode for callers that cannot allocate device
// memory themselves.  The split-context partials go to a file-scope device
// array owned by the library instead of a caller-provided workspace.
// ---------------------------------------------------------------------------
namespace {

// Part of the loaded module: every GPU that loads this library holds these
// PA_FIXED_SCRATCH_BYTES until the process exits.  Host code must not use the
// symbol's name as an address (it is a host-side stand-in); it takes the
// device address from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_fixed_scratch[PA_FIXED_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_fixed_scratch_mutex;
// One cached address per device, valid for the context it was looked up in:
// a context that is torn down (cudaDeviceReset, or the primary context
// released) and created again loads the module again, and the array may then
// sit at another address.  Context ids are never reused within a process.
struct FixedScratchEntry {
  unsigned long long ctx_id;
  void* addr;
};
FixedScratchEntry g_fixed_scratch_cache[kMaxDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// The unique id of the calling thread's current context, or 0 when it has
// none yet (driver entry points looked up once through the runtime).
pa_status current_context_id(unsigned long long* id) {
  static std::atomic<CtxGetCurrentFn> get_current{nullptr};
  static std::atomic<CtxGetIdFn> get_id{nullptr};
  CtxGetCurrentFn cur = get_current.load();
  CtxGetIdFn gid = get_id.load();
  if (!cur || !gid) {
    void* p1 = nullptr;
    void* p2 = nullptr;
    cudaDriverEntryPointQueryResult q1, q2;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p1, cudaEnableDefault, &q1) != cudaSuccess ||
        q1 != cudaDriverEntryPointSuccess || !p1 ||
        cudaGetDriverEntryPoint("cuCtxGetId", &p2, cudaEnableDefault, &q2) != cudaSuccess ||
        q2 != cudaDriverEntryPointSuccess || !p2)
      return fail(PA_ERR_CUDA, "decode_fixed_scratch: the driver's context queries are unavailable");
    cur = reinterpret_cast<CtxGetCurrentFn>(p1);
    gid = reinterpret_cast<CtxGetIdFn>(p2);
    get_current.store(cur);
    get_id.store(gid);
  }
  CUcontext ctx = nullptr;
  *id = 0;
  if (cur(&ctx) != CUDA_SUCCESS) return fail(PA_ERR_CUDA, "decode_fixed_scratch: cuCtxGetCurrent failed");
  if (ctx && gid(ctx, id) != CUDA_SUCCESS) return fail(PA_ERR_CUDA, "decode_fixed_scratch: cuCtxGetId failed");
  return PA_OK;
}

// Device address of g_fixed_scratch in the current device's current context,
// looked up once per (device, context), with that device current, and cached.
pa_status fixed_scratch_address(void** addr) {
  int dev = -1;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return fail(PA_ERR_CUDA, "decode_fixed_scratch: cudaGetDevice: %s", cudaGetErrorString(err));
  if (dev < 0 || dev >= kMaxDevices) return fail(PA_ERR_UNSUPPORTED, "decode_fixed_scratch: device %d", dev);
  unsigned long long ctx_id = 0;
  pa_status st = current_context_id(&ctx_id);
  if (st != PA_OK) return st;
  std::lock_guard<std::mutex> lock(g_fixed_scratch_mutex);
  FixedScratchEntry& e = g_fixed_scratch_cache[dev];
  if (ctx_id == 0 || !e.addr || e.ctx_id != ctx_id) {
    void* p = nullptr;
    err = cudaGetSymbolAddress(&p, g_fixed_scratch);  // also makes the runtime's context current
    if (err != cudaSuccess || !p)
      return fail(PA_ERR_CUDA, "decode_fixed_scratch: cudaGetSymbolAddress: %s", cudaGetErrorString(err));
    if (ctx_id == 0) {
      st = current_context_id(&ctx_id);
      if (st != PA_OK) return st;
    }
    e.addr = p;
    e.ctx_id = ctx_id;
  }
  *addr = e.addr;
  return PA_OK;
}

}  // namespace

extern "C" pa_status pa_decode_fixed_scratch(const void* q, const void* key_cache, const void* value_cache,
                                             const int32_t* block_tables, int32_t max_blocks_per_seq,
                                             const int32_t* context_lens, int32_t num_seqs, int32_t num_q_heads,
                                             int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                             int32_t num_blocks, float scale, void* out, pa_dtype dtype,
                                             int32_t* dev_status, void* stream) {
  // Calls that need no scratch (no sequences) or that pa_decode would reject
  // anyway are handed to it without the one-time set-up.
  if (num_seqs <= 0 || max_blocks_per_seq <= 0 || block_size <= 0 || num_q_heads <= 0 || head_dim <= 0)
    return pa_decode(q, key_cache, value_cache, block_tables, max_blocks_per_seq, context_lens, num_seqs,
                     num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, scale, out, dtype, nullptr, 0,
                     dev_status, stream);
  const size_t need = pa_decode_workspace_size(num_seqs, num_q_heads, head_dim,
                                               (int64_t)max_blocks_per_seq * block_size);
  if (need > (size_t)PA_FIXED_SCRATCH_BYTES)
    return fail(PA_ERR_INVALID,
                "decode_fixed_scratch: this call needs %zu bytes of scratch, more than the fixed %zu-byte array; "
                "use pa_decode with a caller-provided workspace",
                need, (size_t)PA_FIXED_SCRATCH_BYTES);
  void* scratch = nullptr;
  pa_status st = fixed_scratch_address(&scratch);  // first call in a context: the one-time set-up
  if (st != PA_OK) return st;
  return pa_decode(q, key_cache, value_cache, block_tables, max_blocks_per_seq, context_lens, num_seqs, num_q_heads,
                   num_kv_heads, head_dim, block_size, num_blocks, scale, out, dtype, scratch,
                   (size_t)PA_FIXED_SCRATCH_BYTES, dev_status, stream);
}

extern "C" pa_status pa_decode_shared_prefix(const void* q, const void* key_cache, const void* value_cache,
                                             const int32_t* block_tables, int32_t max_blocks_per_seq,
                                             const int32_t* context_lens, int32_t num_seqs, int32_t num_q_heads,
                                             int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                             int32_t num_blocks, float scale, void* out, pa_dtype dtype,
                                             void* workspace, size_t workspace_bytes, const int32_t* first_partition,
                                             const int32_t* chunks, int32_t num_chunks, const int32_t* members,
                                             int32_t num_members, int32_t max_shared_partitions,
                                             int32_t min_shared_partitions, int32_t* dev_status, void* stream) {
  DecodeArgs a;
  int partitions = 0;
  pa_status st = prepare_decode(q, key_cache, value_cache, block_tables, max_blocks_per_seq, context_lens, num_seqs,
                                num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, scale, out, dtype,
                                workspace, workspace_bytes, dev_status, a, partitions);
  if (st != PA_OK || num_seqs == 0) return st;
  if (num_chunks < 0 || num_members < 0 || max_shared_partitions < 0 || min_shared_partitions < 0 ||
      min_shared_partitions > max_shared_partitions)
    return fail(PA_ERR_INVALID, "decode_shared_prefix: bad plan sizes");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool joint = (dtype == PA_BF16 || dtype == PA_F16) && (head_dim == 64 || head_dim == 128) &&
                     block_size % 16 == 0 && a.group <= PA_PREFIX_QUERIES_PER_CTA && partitions > 1 &&
                     num_chunks > 0 && num_members > 0 && max_shared_partitions > 0 && first_partition && chunks &&
                     members;
  const int choice = g_shared_kernel.load();
  // The balanced kernel's walk counts 64-token steps per kv head in 32 bits: an
  // upper bound of the call's units must stay below kSegMaxUnits.
  const int64_t unit_bound =
      (int64_t)num_kv_heads * ((int64_t)num_chunks * (max_shared_partitions * 8 + 3) +
                               (int64_t)num_seqs * ((int64_t)max_blocks_per_seq * block_size / 64 + 1 + 2));
  // AUTO takes the balanced kernel when the members' own tokens are a small share
  // of the shared work (beams over a long prompt): it then runs them itself at
  // little cost.  Many long private tails of few rows each (many sequences over a
  // common prompt) run better in the per-sequence kernel beside the per-partition
  // joint kernel.
  const int64_t tail_bound = (int64_t)num_members * std::max<int64_t>(
      0, (int64_t)max_blocks_per_seq * block_size - (int64_t)min_shared_partitions * kPartition);
  const bool tails_light = 8 * tail_bound <= (int64_t)num_chunks * max_shared_partitions * kPartition;
  if (joint && unit_bound < kSegMaxUnits &&
      ((choice == PA_SHARED_PREFIX_AUTO && tails_light) || choice == PA_SHARED_PREFIX_TCGEN05)) {
    // Balanced tcgen05 kernel: the groups' shared partitions and their members'
    // own tokens in one grid; a per-sequence kernel only for the sequences outside
    // every group (run first, so that the joint grid fills the SMs it leaves).
    if (!aligned16(chunks)) return fail(PA_ERR_INVALID, "decode_shared_prefix: chunks must be 16-byte aligned");
    const bool others = num_members < num_seqs;
    if (others) {
      DecodeArgs ap = a;
      ap.first_partition = first_partition;
      ap.skip_members = 1;
      ap.partition_base = 0;
      st = launch_partitions(ap, dtype, head_dim, num_seqs, partitions, s);
      if (st != PA_OK) return st;
    }
    cudaError_t err;
    if (head_dim == 64)
      err = dtype == PA_BF16 ? launch_shared_seg<__nv_bfloat16, 64>(a, dtype, num_chunks, chunks, members, num_members,
                                                                     first_partition, num_seqs, others, s)
                             : launch_shared_seg<__half, 64>(a, dtype, num_chunks, chunks, members, num_members,
                                                             first_partition, num_seqs, others, s);
    else
      err = dtype == PA_BF16 ? launch_shared_seg<__nv_bfloat16, 128>(a, dtype, num_chunks, chunks, members, num_members,
                                                                      first_partition, num_seqs, others, s)
                             : launch_shared_seg<__half, 128>(a, dtype, num_chunks, chunks, members, num_members,
                                                              first_partition, num_seqs, others, s);
    if (err != cudaSuccess) return fail(PA_ERR_CUDA, "decode shared-prefix kernel: %s", cudaGetErrorString(err));
    return launch_reduce_any(a, dtype, head_dim, num_seqs, s, /*dependent=*/true, /*sparse=*/1);
  }
  if (joint && unit_bound < kSegMaxUnits && choice == PA_SHARED_PREFIX_AUTO) {
    // Tail-heavy plans: the balanced kernel on the shared lanes only, then the
    // per-sequence kernel on every partition from each sequence's first_partition
    // (a programmatic dependent: its CTAs take the SMs the joint grid's CTAs
    // leave), then the sparse merge.
    if (!aligned16(chunks)) return fail(PA_ERR_INVALID, "decode_shared_prefix: chunks must be 16-byte aligned");
    cudaError_t err;
    if (head_dim == 64)
      err = dtype == PA_BF16 ? launch_shared_seg<__nv_bfloat16, 64>(a, dtype, num_chunks, chunks, members, num_members,
                                                                     first_partition, num_seqs, false, s, false)
                             : launch_shared_seg<__half, 64>(a, dtype, num_chunks, chunks, members, num_members,
                                                             first_partition, num_seqs, false, s, false);
    else
      err = dtype == PA_BF16 ? launch_shared_seg<__nv_bfloat16, 128>(a, dtype, num_chunks, chunks, members, num_members,
                                                                      first_partition, num_seqs, false, s, false)
                             : launch_shared_seg<__half, 128>(a, dtype, num_chunks, chunks, members, num_members,
                                                              first_partition, num_seqs, false, s, false);
    if (err != cudaSuccess) return fail(PA_ERR_CUDA, "decode shared-prefix kernel: %s", cudaGetErrorString(err));
    DecodeArgs ap = a;
    ap.first_partition = first_partition;
    ap.partition_base = min_shared_partitions < partitions - 1 ? min_shared_partitions : partitions - 1;
    st = launch_partitions(ap, dtype, head_dim, num_seqs, partitions, s, /*dependent=*/true);
    if (st != PA_OK) return st;
    return launch_reduce_any(a, dtype, head_dim, num_seqs, s, /*dependent=*/true, /*sparse=*/1);
  }
  if (joint) {
    if (!aligned16(chunks)) return fail(PA_ERR_INVALID, "decode_shared_prefix: chunks must be 16-byte aligned");
    dim3 grid(num_chunks, num_kv_heads, max_shared_partitions < partitions ? max_shared_partitions : partitions);
    const cudaError_t err =
        dtype == PA_BF16
            ? launch_shared_dim<__nv_bfloat16>(a, head_dim, grid, chunks, members, num_members, num_seqs, dtype, s)
            : launch_shared_dim<__half>(a, head_dim, grid, chunks, members, num_members, num_seqs, dtype, s);
    if (err != cudaSuccess) return fail(PA_ERR_CUDA, "decode shared-prefix kernel: %s", cudaGetErrorString(err));
    a.first_partition = first_partition;
    // Partitions below every sequence's first_partition need no per-sequence CTA.
    a.partition_base = min_shared_partitions < partitions - 1 ? min_shared_partitions : partitions - 1;
  }
  st = launch_partitions(a, dtype, head_dim, num_seqs, partitions, s, /*dependent=*/joint);
  if (st != PA_OK || partitions <= 1) return st;
  return launch_reduce_any(a, dtype, head_dim, num_seqs, s);
}

// GQA decode with block routing and the zero-order tail.
//
// SPLA §1-2 notes that decoding is bound by loading the KV cache and keeps
// the IO profile of sparse decoding: only the selected blocks are read token
// by token; every other block is represented by its precomputed statistics.
// Up to four launches on the caller's stream, each started early by
// programmatic dependent launch:
//   A. the statistics pass (decode_stats_kernel for float32 statistics,
//        decode_stats_mma_kernel for bf16 ones, decode_stats_tc_kernel in
//        decode_tc.cu for bf16 ones with d = 128): one pass over kmean, kvar
//        (and the value means), each read once: the SPLA §2.1 score of every
//        block for each query head, summed over the GQA group (logsumexp)
//        -> scores, and the PISA zero-order term of EVERY block -> per-segment
//        partial states (max, sum, acc) per query head;
//   B. decode_topk_kernel   top-k per (sequence, KV head) -> block_idx
//        (skipped when the tensor-core statistics pass selected the blocks);
//   C. decode_exact_kernel  the selected blocks token by token (exact online
//        softmax) -> per-segment partial states;
//   D. decode_combine_kernel  merges A's states, subtracts each selected
//        block's own zero-order term (the subtraction form of SPLA §2.2
//        applied to PISA's tail; it cannot cancel below zero because
//        Σ_n e^{x_n} ≥ B e^{mean x} for every block), merges C's states -> o.
// A and C are persistent streaming kernels: each CTA walks a list of stages
// staged into shared memory with cp.async (or TMA), several stages deep, so
// the HBM stays busy while the previous stage is reduced.
#include <cuda.h>

#include <mutex>
#include <utility>
#include <vector>

#include "topk.cuh"

namespace sa {
namespace {

constexpr int kDecThreads = 256;
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kMaxGroup = 8;

// A: a stage is 32 blocks of statistics (kmean, kvar, vsum rows); a segment
// is kSegA stages (one partial state per segment and query head)
constexpr int kStageBlocksA = 32;
constexpr int kSegA = 4;
constexpr int kRingA = 2;
// C: a stage is 128 selected tokens of K and V (two 64-token halves, each
// inside one selected block); a segment is kSegC stages
constexpr int kStageTokC = 128;
constexpr int kSegC = 4;
constexpr int kRingC = 3;
// segments per CTA whose block indices are staged in shared memory (later
// segments read theirs from global memory)
constexpr int kItabSegs = 64;

struct DecodeLayout {
  size_t scores_off, idx_off, parta_off, partc_off, partr_off, total;
  int nsegA, nsegC;
};

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

DecodeLayout decode_layout(const sa_decode_shape& s, int topk) {
  DecodeLayout L;
  const int nb = s.N / s.block;
  L.nsegA = (nb + kStageBlocksA * kSegA - 1) / (kStageBlocksA * kSegA);
  L.nsegC = (int)(((long)topk * s.block + kStageTokC * kSegC - 1) / (kStageTokC * kSegC));
  const size_t part = (size_t)(s.d + 2) * sizeof(float);
  L.scores_off = 0;
  L.idx_off = align256((size_t)s.B * s.Hkv * nb * sizeof(float));
  L.parta_off = L.idx_off + align256((size_t)s.B * s.Hkv * (topk > 0 ? topk : 1) * sizeof(int32_t));
  L.partc_off = L.parta_off + align256((size_t)s.B * s.Hq * (L.nsegA > 0 ? L.nsegA : 1) * part);
  L.total = L.partc_off + align256((size_t)s.B * s.Hq * (L.nsegC > 0 ? L.nsegC : 1) * part);
  // residual linear tail: per (query head, exact segment) the selected
  // tokens' Σ (φ(q)·φ(k_n)) v_n, over the statistics pass's partial states
  // (which that tail does not read) when they fit there, else appended
  const size_t partr = (size_t)s.B * s.Hq * (L.nsegC > 0 ? L.nsegC : 1) * s.d * sizeof(float);
  const size_t parta = (size_t)s.B * s.Hq * (L.nsegA > 0 ? L.nsegA : 1) * part;
  if (partr <= parta) {
    L.partr_off = L.parta_off;
  } else {
    L.partr_off = L.total;
    L.total += align256(partr);
  }
  return L;
}

// Device-side error word of the decode kernels: set when a bounded wait gives
// up; sa_device_error() reads and clears it with the attention kernels' word.
static __device__ unsigned int g_decode_error = 0;
constexpr long long kDecWaitCycles = 4000000000ll;   // ~2 s: far above any real wait

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void dbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void dbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
// Waits for the phase of parity `parity`; false after kDecWaitCycles (the
// error word is set).
__device__ __forceinline__ bool dbar_wait(uint32_t bar, uint32_t parity) {
  const long long t0 = clock64();
  for (;;) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    if (done) return true;
    if (clock64() - t0 > kDecWaitCycles) {
      atomicOr(&g_decode_error, 1u);
      return false;
    }
  }
}
// One contiguous global -> shared copy of `bytes` (16-byte aligned, a
// multiple of 16) completing on `bar`.
__device__ __forceinline__ void bulk_copy(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(dst), "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

// 16-byte cp.async reading `src_bytes` (16 or 0) and zero-filling the rest
__device__ __forceinline__ void cp_async16z(void* smem_dst, const void* gsrc, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"((uint32_t)__cvta_generic_to_shared(smem_dst)),
               "l"(gsrc), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ uint32_t pack2bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// SPLA's feature map φ = exp on both halves of a packed bf16 pair, rounded
// back to bf16 (the same rounding as the all-token state in sa_block_pool)
__device__ __forceinline__ uint32_t phi_bf16x2(uint32_t x) {
  const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&x));
  return pack2bf16(phi_exp(f.x), phi_exp(f.y));
}

// Partial online-softmax state of one query head in a warp: log2-domain max,
// lane-partial sum, and the lane's 4 channels (lane = channel group).
struct HeadState {
  float m, l, acc[4];
};

// Writes the warp's state (lane sums reduced) to out[0..D+2) (D = 128: 4
// channels per lane; D = 64: lanes 0..15 hold 4 channels each).
template <int D>
__device__ __forceinline__ void head_store(const HeadState& S, float* out, int lane) {
  const float l = warp_sum(S.l);
  if (lane == 0) {
    out[0] = S.m;
    out[1] = l;
  }
  if (lane * 4 < D) {
#pragma unroll
    for (int c = 0; c < 4; ++c) out[2 + lane * 4 + c] = S.acc[c];
  }
}

// ---- A. statistics pass --------------------------------------------------
// Two CTAs of 8 warps per SM.  A stage (32 blocks of kmean, kvar and vsum
// rows, 48 KB for d = 128) lands in shared memory by three bulk copies
// issued by one thread; warp w takes blocks [4w, 4w + 4) of it.  Lane = a group of d/32 channels: it holds
// s log2e q and ½ s² q² of the group's channels for all G heads in
// registers and reads each stats row as one contiguous 512-byte row, so a
// row costs four shared-memory wavefronts and is read by one warp only.
// A batch of 16/G blocks gives each lane 32 partial sums (q·k̄ and
// ½ s² Σ q² Var for each (block, head)); a reduce-scatter over the warp
// (31 shuffles) leaves value v in lane v, fully summed.  The zero-order
// terms of the batch then enter the warp's online state of each head
// (max, sum, numerator channels of the lane); the four warps' states are
// merged once per segment.
constexpr int kThrA = 256;

// channels [lane CPL, lane CPL + CPL) of a shared-memory row, or zeros
template <int CPL>
__device__ __forceinline__ void load_lane(float (&r)[CPL], const float* row, int lane, bool ok) {
  if constexpr (CPL == 4) {
    const float4 x = ok ? *reinterpret_cast<const float4*>(row + lane * 4) : make_float4(0.f, 0.f, 0.f, 0.f);
    r[0] = x.x;
    r[1] = x.y;
    r[2] = x.z;
    r[3] = x.w;
  } else {
    const float2 x = ok ? *reinterpret_cast<const float2*>(row + lane * 2) : make_float2(0.f, 0.f);
    r[0] = x.x;
    r[1] = x.y;
  }
}
template <int CPL>
__device__ __forceinline__ void load_lane(float (&r)[CPL], const __nv_bfloat16* row, int lane, bool ok) {
  if constexpr (CPL == 4) {
    const uint2 x = ok ? *reinterpret_cast<const uint2*>(row + lane * 4) : make_uint2(0u, 0u);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&x.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&x.y));
    r[0] = a.x;
    r[1] = a.y;
    r[2] = b.x;
    r[3] = b.y;
  } else {
    const uint32_t x = ok ? *reinterpret_cast<const uint32_t*>(row + lane * 2) : 0u;
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&x));
    r[0] = a.x;
    r[1] = a.y;
  }
}

// Ring depth of the statistics pass: the same bytes in flight per CTA for
// float32 and bf16 statistics (bf16 stages are half as large)
template <typename TS>
constexpr int ring_a() { return sizeof(TS) == 4 ? kRingA : 2 * kRingA - 1; }

constexpr int kWarpBlocksA = kStageBlocksA / (kThrA / 32);   // blocks of a stage per warp

// ZT: the zero-order tail is wanted (its value sums are copied and its
// online state kept); without it the pass only scores the blocks.
// TS: element type of the statistics, float (kmean, kvar, vsum) or bf16
// (kmean, kvar and the value means vsum / blk); vmul turns a row of the
// third array into the block's value mean (1 / blk for sums, 1 for means).
template <int D, int G, bool ZT, typename TS>
__global__ void __launch_bounds__(kThrA, 2)
decode_stats_kernel(const __nv_bfloat16* __restrict__ q, const TS* __restrict__ kmean, const TS* __restrict__ kvar,
                    const TS* __restrict__ vrow, float vmul, int Hq, int Hkv, int nb, int blk, float scale,
                    int nsegA, int npairs, float* __restrict__ scores, float* __restrict__ parta) {
  constexpr int CPL = D / 32;                        // channels per lane
  constexpr int NBT = 16 / G;                        // blocks per batch: NBT x G x 2 = 32 sums
  constexpr int kBatches = (kWarpBlocksA + NBT - 1) / NBT;
  constexpr int RING = ring_a<TS>();
  constexpr uint32_t kRowB = D * sizeof(TS);         // bytes per stats row
  constexpr uint32_t kArrB = kStageBlocksA * kRowB;  // one array of one stage
  constexpr uint32_t kStageB = 3 * kArrB;
  constexpr int kWarps = kThrA / 32;
  extern __shared__ __align__(16) uint8_t dsm[];
  float* mg = reinterpret_cast<float*>(dsm);                 // [warps][G][D + 2] segment merge
  uint64_t* full = reinterpret_cast<uint64_t*>(dsm + sizeof(float) * kWarps * G * (D + 2));   // [RING]
  uint8_t* ring = reinterpret_cast<uint8_t*>(full + 2 * RING);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nstage_pair = (nb + kStageBlocksA - 1) / kStageBlocksA;
  const int total_segs = npairs * nsegA;
  const float bias2 = log2f((float)blk);
  const int hl = (lane >> 1) % G, jbl = (lane >> 1) / G;   // the (block, head) of the sum lane ends with

  // the CTA's stage sequence: its segments in order, each segment's stages
  auto seg_of = [&](int k_seg) { return (int)blockIdx.x + k_seg * (int)gridDim.x; };
  auto stages_in = [&](int seg) { return min(kSegA, nstage_pair - (seg % nsegA) * kSegA); };
  // thread 0 copies stage `sub` of segment `seg` into ring slot `slot`: the
  // stage's rows of each array are contiguous, one bulk copy per array
  auto issue = [&](int seg, int sub, int slot) {
    const int pair = seg / nsegA, sseg = seg % nsegA;
    const int j0 = (sseg * kSegA + sub) * kStageBlocksA;
    const uint32_t bytes = (uint32_t)min(kStageBlocksA, nb - j0) * kRowB;
    const size_t goff = ((size_t)pair * nb + j0) * D;
    const uint32_t dst = smem_addr(ring + slot * kStageB), fb = smem_addr(full + slot);
    // the slot's previous contents were read by generic loads before the
    // barrier that precedes this call; order them before the async writes
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    dbar_expect_tx(fb, (ZT ? 3 : 2) * bytes);
    bulk_copy(dst, kmean + goff, bytes, fb);
    bulk_copy(dst + kArrB, kvar + goff, bytes, fb);
    if (ZT) bulk_copy(dst + 2 * kArrB, vrow + goff, bytes, fb);
  };

  if (seg_of(0) >= total_segs) return;
  if (tid == 0) {
    for (int r = 0; r < RING; ++r) dbar_init(smem_addr(full + r), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  int cur_seg_k = 0, cur_sub = 0;
  int pf_seg_k = 0, pf_sub = 0, pf_slot = 0;
  int issued = 0, consumed = 0;   // stages copied / used (ring phases)
  auto pf_valid = [&]() { return seg_of(pf_seg_k) < total_segs; };
  auto pf_advance = [&]() {
    if (++pf_sub >= stages_in(seg_of(pf_seg_k))) {
      pf_sub = 0;
      ++pf_seg_k;
    }
  };
  for (int r = 0; r < RING - 1; ++r) {
    if (pf_valid()) {
      if (tid == 0) issue(seg_of(pf_seg_k), pf_sub, pf_slot);
      ++issued;
      pf_advance();
    }
    pf_slot = (pf_slot + 1) % RING;
  }

  float qv[G][CPL], wv[G][CPL];   // s log2e q and ½ s² q² of this lane's channels
  float m[G], l[G], acc[G][CPL];  // the warp's online state per head (m, l replicated in all lanes)
  int cur_pair = -1;
  int slot = 0;
  while (seg_of(cur_seg_k) < total_segs) {
    const int seg = seg_of(cur_seg_k);
    const int pair = seg / nsegA, sseg = seg % nsegA;
    const int b = pair / Hkv, kh = pair % Hkv;
    if (cur_sub == 0) {
      if (pair != cur_pair) {
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
          for (int c = 0; c < CPL; ++c) {
            const float v = __bfloat162float(q[((size_t)b * Hq + kh * G + h) * D + lane * CPL + c]);
            qv[h][c] = scale * kLog2e * v;
            wv[h][c] = 0.5f * scale * scale * v * v;
          }
        cur_pair = pair;
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        m[h] = -INFINITY;
        l[h] = 0.f;
#pragma unroll
        for (int c = 0; c < CPL; ++c) acc[h][c] = 0.f;
      }
    }
    // prefetch one more stage (its slot was released by the previous
    // stage's closing barrier), then wait for the current one
    if (pf_valid()) {
      if (tid == 0) issue(seg_of(pf_seg_k), pf_sub, pf_slot);
      ++issued;
      pf_advance();
    }
    pf_slot = (pf_slot + 1) % RING;
    const bool landed = dbar_wait(smem_addr(full + slot), (consumed / RING) & 1);
    ++consumed;
    if (!__syncthreads_and(landed)) break;

    const uint8_t* stg = ring + slot * kStageB;
    const TS* km = reinterpret_cast<const TS*>(stg);
    const TS* kv = reinterpret_cast<const TS*>(stg + kArrB);
    const TS* vs = reinterpret_cast<const TS*>(stg + 2 * kArrB);
    const int j0 = (sseg * kSegA + cur_sub) * kStageBlocksA;
    const int rows = min(kStageBlocksA, nb - j0);

#pragma unroll
    for (int bi = 0; bi < kBatches; ++bi) {
      const int jfirst = warp * kWarpBlocksA + bi * NBT;   // stage row of the batch's block 0
      // partial sums, value index (jb G + h) 2 + kind (kind 0: q·k̄, 1: Σ q² Var)
      float v[32];
#pragma unroll
      for (int jb = 0; jb < NBT; ++jb) {
        const int jj = jfirst + jb;
        float a[CPL], w[CPL];
        const bool ok = jb < kWarpBlocksA - bi * NBT && jj < rows;
        load_lane<CPL>(a, km + jj * D, lane, ok);
        load_lane<CPL>(w, kv + jj * D, lane, ok);
#pragma unroll
        for (int h = 0; h < G; ++h) {
          float s1 = a[0] * qv[h][0], s2 = w[0] * wv[h][0];
#pragma unroll
          for (int c = 1; c < CPL; ++c) {
            s1 = fmaf(a[c], qv[h][c], s1);
            s2 = fmaf(w[c], wv[h][c], s2);
          }
          v[(jb * G + h) * 2] = s1;
          v[(jb * G + h) * 2 + 1] = s2;
        }
      }
      // reduce-scatter: after the step of offset o, a lane keeps the half of
      // its 2o values selected by bit o of its index; value `lane` remains
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) {
        const bool up = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < o; ++i) {
          const float send = up ? v[i] : v[i + o];
          const float keep = up ? v[i + o] : v[i];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
      }
      const float other = __shfl_xor_sync(0xffffffffu, v[0], 1);
      const float d1 = (lane & 1) ? other : v[0];           // s log2e q·k̄
      const float d2 = (lane & 1) ? v[0] : other;           // ½ s² Σ q² Var
      const int jj = jfirst + jbl;
      const bool live = (lane & 1) == 0 && jbl < kWarpBlocksA - bi * NBT && jj < rows;
      // group score of the block: logsumexp over its G heads (lanes 2 apart)
      const float ls = live ? d1 * kLn2 + log1pf(d2) : -INFINITY;
      float mx = ls;
#pragma unroll
      for (int o = 2; o < 2 * G; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      float se = live ? expf(ls - mx) : 0.f;
#pragma unroll
      for (int o = 2; o < 2 * G; o <<= 1) se += __shfl_xor_sync(0xffffffffu, se, o);
      if (live && hl == 0) scores[(size_t)pair * nb + j0 + jj] = mx + logf(se);
      if (!ZT) continue;
      // zero-order term: log2 weight of the pseudo-key (value vsum / B)
      const float x = live ? d1 + bias2 : -INFINITY;
      float bm = x;
#pragma unroll
      for (int o = 2 * G; o < 32; o <<= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o));
      float mnew[G], corr[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        mnew[h] = fmaxf(m[h], __shfl_sync(0xffffffffu, bm, 2 * h));
        corr[h] = m[h] == -INFINITY ? 0.f : fast_exp2(m[h] - mnew[h]);
      }
      float mown = mnew[0];
#pragma unroll
      for (int h = 1; h < G; ++h)
        if (hl == h) mown = mnew[h];
      const float p = (live && mown != -INFINITY) ? fast_exp2(x - mown) : 0.f;
      float ps = p;
#pragma unroll
      for (int o = 2 * G; o < 32; o <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
#pragma unroll
      for (int h = 0; h < G; ++h) {
        l[h] = l[h] * corr[h] + __shfl_sync(0xffffffffu, ps, 2 * h);
        m[h] = mnew[h];
#pragma unroll
        for (int c = 0; c < CPL; ++c) acc[h][c] *= corr[h];
      }
#pragma unroll
      for (int jb = 0; jb < NBT; ++jb) {
        const int jr = jfirst + jb;
        const bool ok = jb < kWarpBlocksA - bi * NBT && jr < rows;
        float vv[CPL];
        load_lane<CPL>(vv, vs + jr * D, lane, ok);
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float pw = __shfl_sync(0xffffffffu, p, (jb * G + h) * 2) * vmul;
#pragma unroll
          for (int c = 0; c < CPL; ++c) acc[h][c] = fmaf(pw, vv[c], acc[h][c]);
        }
      }
    }
    slot = (slot + 1) % RING;
    // end of segment: merge the warps' states per head and write them
    const bool seg_end = ++cur_sub >= stages_in(seg);
    if (ZT && seg_end) {
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float* mw = mg + (warp * G + h) * (D + 2);
        if (lane == 0) {
          mw[0] = m[h];
          mw[1] = l[h];
        }
#pragma unroll
        for (int c = 0; c < CPL; ++c) mw[2 + lane * CPL + c] = acc[h][c];
      }
    }
    __syncthreads();   // the ring slot is reused by the next prefetch; the merge rows are complete
    if (seg_end) {
      for (int x = tid; ZT && x < G * D; x += kThrA) {
        const int h = x / D, c = x % D;
        float M = -INFINITY;
#pragma unroll
        for (int w2 = 0; w2 < kWarps; ++w2) M = fmaxf(M, mg[(w2 * G + h) * (D + 2)]);
        float L = 0.f, A = 0.f;
        if (M != -INFINITY) {
#pragma unroll
          for (int w2 = 0; w2 < kWarps; ++w2) {
            const float* mw = mg + (w2 * G + h) * (D + 2);
            if (mw[0] == -INFINITY) continue;
            const float f = fast_exp2(mw[0] - M);
            L = fmaf(mw[1], f, L);
            A = fmaf(mw[2 + c], f, A);
          }
        }
        float* out = parta + (((size_t)b * Hq + kh * G + h) * nsegA + sseg) * (D + 2);
        if (c == 0) {
          out[0] = M;
          out[1] = L;
        }
        out[2 + c] = A;
      }
      if (ZT) __syncthreads();   // the merge rows are rewritten at the next segment end
      cur_sub = 0;
      ++cur_seg_k;
    }
  }
  // after a give-up, let the copies still in flight land before exiting
  if (tid == 0)
    for (int q = consumed; q < issued; ++q) dbar_wait(smem_addr(full + q % RING), (q / RING) & 1);
}

// ---- B. top-k ------------------------------------------------------------
// The top-k of each (sequence, KV head) row: radix_topk_cta (topk.cuh).
__global__ void __launch_bounds__(kDecThreads)
decode_topk_kernel(const float* __restrict__ scores, int nb, int topk, int32_t* __restrict__ idx) {
  pdl_wait();
  pdl_trigger();
  __shared__ RadixTopkSmem sm;
  const int pair = blockIdx.x;
  radix_topk_cta<kDecThreads>(scores + (size_t)pair * nb, nb, topk, idx + (size_t)pair * topk, sm);
}

// ---- C. exact pass over the selected blocks --------------------------------
// A stage is 128 selected tokens, two 64-token halves of selected blocks (K
// and V rows staged by cp.async with the 16-byte chunks of row r stored at
// chunk ^ (r & 7), so ldmatrix reads are free of bank conflicts).  Warp w
// takes tokens [16w, 16w + 16) of each stage and runs the small contractions
// on mma.sync
// (m16n8k16, bf16 in, fp32 accumulate): S = Q Kᵀ with the group's g <= 8
// query heads as the MMA rows, then O += P V.  Each warp keeps an online
// softmax state per head; at the end of a segment the eight warps' states are
// merged and one partial state per head is written.  The selected block
// indices of all the CTA's segments are staged in shared memory once, so the
// copy issue of a stage does not wait on a global load.
__device__ __forceinline__ void mma16816_full(float (&d)[4], uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}
// The same MMA when rows 8-15 of A are zero: only d0, d1 (row lane / 4) are
// kept; the other two outputs go to scratch registers.
__device__ __forceinline__ void mma16816_top(float (&d)[2], uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
  float x2, x3;
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%10,%10};"
      : "+f"(d[0]), "+f"(d[1]), "=f"(x2), "=f"(x3)
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1), "f"(0.f));
  (void)x2;
  (void)x3;
}
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// floats of the exact pass's merge rows ([g][8 warps][D + 2]), rounded up to
// 128 bytes; sized by the group rather than its maximum so that the pass
// leaves room on the SM for a combine CTA, which then runs its prologue
// while the pass streams
__host__ __device__ constexpr int exact_merge_floats(int g, int D) {
  return (kDecWarps * g * (D + 2) + 31) & ~31;
}

template <int D, bool RLA>
__global__ void __launch_bounds__(kDecThreads, 1)
decode_exact_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ Kc,
                    const __nv_bfloat16* __restrict__ Vc, int Hq, int Hkv, int N, int blk,
                    const int32_t* __restrict__ idx, int topk, float scale, int nsegC, int npairs,
                    float* __restrict__ partc, float* __restrict__ partr) {
  pdl_wait();
  pdl_trigger();
  constexpr int CH = D / 8;                         // 16-byte chunks per bf16 row
  constexpr int NT = D / 8;                         // n-tiles of 8 channels
  constexpr int KS = D / 16;                        // k steps of 16 channels
  constexpr uint32_t kRowB = D * 2;
  constexpr uint32_t kArrB = kStageTokC * kRowB;    // K (or V) of one stage
  constexpr uint32_t kStageB = 2 * kArrB;
  constexpr int kSegBlocksMax = kSegC * kStageTokC / 64;   // blocks of a segment (blk >= 64)
  extern __shared__ __align__(16) uint8_t dsm[];
  const int g = Hq / Hkv;
  float* mg = reinterpret_cast<float*>(dsm);                         // [g][8 warps][D + 2] merge
  int* itab = reinterpret_cast<int*>(mg + exact_merge_floats(g, D));   // [segments][blocks]
  uint8_t* ring = reinterpret_cast<uint8_t*>(itab + kItabSegs * kSegBlocksMax);
  const uint32_t ring_s = (uint32_t)__cvta_generic_to_shared(ring);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int tok_pair = topk * blk;                  // exact tokens of one (sequence, KV head)
  const int nstage_pair = (tok_pair + kStageTokC - 1) / kStageTokC;   // the last may hold 64
  const int total_segs = npairs * nsegC;
  const float scale2 = scale * kLog2e;
  const int hrow = lane >> 2;                       // MMA row of this thread = query head
  const bool hvalid = hrow < g;

  auto seg_of = [&](int k_seg) { return (int)blockIdx.x + k_seg * (int)gridDim.x; };
  auto stages_in = [&](int seg) { return min(kSegC, nstage_pair - (seg % nsegC) * kSegC); };
  // block slot `sl` (0 .. kSegBlocksMax) of the CTA's k-th segment
  auto block_of = [&](int k, int seg, int sl) {
    const int pair = seg / nsegC, sseg = seg % nsegC;
    const int si = sseg * kSegC * kStageTokC / blk + sl;
    return k < kItabSegs ? itab[k * kSegBlocksMax + sl] : __ldg(idx + (size_t)pair * topk + si);
  };
  // stage `sub` of segment `seg` into ring slot `slot`: two 64-token halves,
  // each inside one selected block; a half past the pair's last selected
  // token is zero-filled (it only occurs as the second half of a last stage)
  auto issue = [&](int k, int seg, int sub, int slot) {
    const int pair = seg / nsegC, sseg = seg % nsegC;
    const int t0 = (sseg * kSegC + sub) * kStageTokC;
    const int ntok = min(kStageTokC, tok_pair - t0);
    const __nv_bfloat16* ks[2];
    const __nv_bfloat16* vsrc[2];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int tin = sub * kStageTokC + 64 * (hh < 1 || 64 < ntok ? hh : 0);   // token offset in the segment
      const size_t off = ((size_t)pair * N + block_of(k, seg, tin / blk) * blk + (tin % blk)) * D;
      ks[hh] = Kc + off;
      vsrc[hh] = Vc + off;
    }
    uint8_t* dst = ring + slot * kStageB;
    for (int o = tid; o < kStageTokC * CH; o += kDecThreads) {
      const int r = o / CH, c = o % CH, hh = r >> 6;
      const uint32_t sw = r * kRowB + ((c ^ (r & 7)) << 4);
      const size_t so = (size_t)(r & 63) * D + 8 * c;
      const uint32_t nbytes = r < ntok ? 16u : 0u;   // 0: zero-fill
      cp_async16z(dst + sw, ks[hh] + so, nbytes);
      cp_async16z(dst + kArrB + sw, vsrc[hh] + so, nbytes);
    }
  };
  if (seg_of(0) >= total_segs) return;
  // the selected blocks of the CTA's first kItabSegs segments
  for (int x = tid; x < kItabSegs * kSegBlocksMax; x += kDecThreads) {
    const int k = x / kSegBlocksMax, sl = x % kSegBlocksMax;
    const int seg = seg_of(k);
    int v = 0;
    if (seg < total_segs) {
      const int pair = seg / nsegC, sseg = seg % nsegC;
      const int si = sseg * kSegC * kStageTokC / blk + sl;
      if (si < topk) v = __ldg(idx + (size_t)pair * topk + si);
    }
    itab[x] = v;
  }
  __syncthreads();
  int pf_seg_k = 0, pf_sub = 0, pf_slot = 0;
  auto pf_valid = [&]() { return seg_of(pf_seg_k) < total_segs; };
  auto prefetch = [&]() {
    if (pf_valid()) {
      issue(pf_seg_k, seg_of(pf_seg_k), pf_sub, pf_slot);
      if (++pf_sub >= stages_in(seg_of(pf_seg_k))) {
        pf_sub = 0;
        ++pf_seg_k;
      }
    }
    cp_async_commit();
    pf_slot = (pf_slot + 1) % kRingC;
  };
  for (int r = 0; r < kRingC - 1; ++r) prefetch();

  uint32_t qa0[KS], qa2[KS];                  // Q A-fragments (rows = heads)
  uint32_t fa0[RLA ? KS : 1], fa2[RLA ? KS : 1];   // φ(Q) A-fragments (residual linear tail)
  float m_run = -INFINITY, l_run = 0.f;
  float o[NT][2];                             // rows 8-15 of the MMA are empty
  float o2[RLA ? NT : 1][2];                  // Σ (φ(q)·φ(k_n)) v_n of the warp's tokens
  int cur_seg_k = 0, cur_sub = 0, cur_pair = -1, slot = 0;
  while (seg_of(cur_seg_k) < total_segs) {
    const int seg = seg_of(cur_seg_k);
    const int pair = seg / nsegC, sseg = seg % nsegC;
    const int b = pair / Hkv, kh = pair % Hkv;
    if (cur_sub == 0) {
      if (pair != cur_pair) {
        const __nv_bfloat16* qrow = q + ((size_t)b * Hq + kh * g + (hvalid ? hrow : 0)) * D;
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
          const uint32_t lo = *reinterpret_cast<const uint32_t*>(qrow + 16 * kk + 2 * (lane & 3));
          const uint32_t hi = *reinterpret_cast<const uint32_t*>(qrow + 16 * kk + 8 + 2 * (lane & 3));
          qa0[kk] = hvalid ? lo : 0u;
          qa2[kk] = hvalid ? hi : 0u;
          if (RLA) {
            fa0[kk] = hvalid ? phi_bf16x2(lo) : 0u;
            fa2[kk] = hvalid ? phi_bf16x2(hi) : 0u;
          }
        }
        cur_pair = pair;
      }
      m_run = -INFINITY;
      l_run = 0.f;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) o[nt][e] = 0.f;
      if (RLA) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int e = 0; e < 2; ++e) o2[RLA ? nt : 0][e] = 0.f;
      }
    }
    prefetch();
    cp_async_wait<kRingC - 1>();
    __syncthreads();

    const uint32_t kbase = ring_s + slot * kStageB, vbase = kbase + kArrB;
    const int ntok = min(kStageTokC, tok_pair - (sseg * kSegC + cur_sub) * kStageTokC);
    const int tb = 16 * warp;                   // this warp's tokens [tb, tb + 16) of the stage
    const int tok0 = tb + (lane & 7), tok1 = tb + 8 + (lane & 7);   // rows this lane addresses
    // S = Q Kᵀ for the warp's two 8-token n-tiles
    float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
    float w0[4] = {0.f, 0.f, 0.f, 0.f}, w1[4] = {0.f, 0.f, 0.f, 0.f};   // φ(q)·φ(k_n)
#pragma unroll
    for (int kp = 0; kp < KS / 2; ++kp) {
      uint32_t kf[4], kg[4];
      const int chunk = 4 * kp + (lane >> 3);
      ldsm_x4(kf, kbase + tok0 * kRowB + ((chunk ^ (tok0 & 7)) << 4));
      ldsm_x4(kg, kbase + tok1 * kRowB + ((chunk ^ (tok1 & 7)) << 4));
      mma16816_full(s0, qa0[2 * kp], qa2[2 * kp], kf[0], kf[1]);
      mma16816_full(s0, qa0[2 * kp + 1], qa2[2 * kp + 1], kf[2], kf[3]);
      mma16816_full(s1, qa0[2 * kp], qa2[2 * kp], kg[0], kg[1]);
      mma16816_full(s1, qa0[2 * kp + 1], qa2[2 * kp + 1], kg[2], kg[3]);
      if (RLA) {
        // the same fragments through the feature map (zero-filled rows give
        // φ = 1, but their V rows are zero)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          kf[e] = phi_bf16x2(kf[e]);
          kg[e] = phi_bf16x2(kg[e]);
        }
        const int kq = RLA ? 2 * kp : 0;
        mma16816_full(w0, fa0[kq], fa2[kq], kf[0], kf[1]);
        mma16816_full(w0, fa0[kq + 1], fa2[kq + 1], kf[2], kf[3]);
        mma16816_full(w1, fa0[kq], fa2[kq], kg[0], kg[1]);
        mma16816_full(w1, fa0[kq + 1], fa2[kq + 1], kg[2], kg[3]);
      }
    }
    // online softmax of the warp's 16 tokens for head hrow (tokens past the
    // stage's valid count are zero-filled rows: masked out)
    const int tj = tb + 2 * (lane & 3);
    const float x0 = tj < ntok ? s0[0] * scale2 : -INFINITY, x1 = tj + 1 < ntok ? s0[1] * scale2 : -INFINITY;
    const float x2 = tj + 8 < ntok ? s1[0] * scale2 : -INFINITY, x3 = tj + 9 < ntok ? s1[1] * scale2 : -INFINITY;
    float tmax = fmaxf(fmaxf(x0, x1), fmaxf(x2, x3));
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 2));
    const float m_new = fmaxf(m_run, tmax);
    const float corr = m_run == -INFINITY ? 0.f : fast_exp2(m_run - m_new);
    const bool on = hvalid && m_new != -INFINITY;
    const float p0 = on && x0 != -INFINITY ? fast_exp2(x0 - m_new) : 0.f;
    const float p1 = on && x1 != -INFINITY ? fast_exp2(x1 - m_new) : 0.f;
    const float p2 = on && x2 != -INFINITY ? fast_exp2(x2 - m_new) : 0.f;
    const float p3 = on && x3 != -INFINITY ? fast_exp2(x3 - m_new) : 0.f;
    l_run = l_run * corr + ((p0 + p1) + (p2 + p3));
    m_run = m_new;
    // P as the A fragment: k 0-7 = the first n-tile's tokens, k 8-15 the second's
    const uint32_t pa0 = pack2bf16(p0, p1), pa2 = pack2bf16(p2, p3);
    const uint32_t wa0 = RLA ? pack2bf16(w0[0], w0[1]) : 0u, wa2 = RLA ? pack2bf16(w1[0], w1[1]) : 0u;
    // O += P V over the 16 tokens
#pragma unroll
    for (int nq = 0; nq < NT / 4; ++nq) {
      uint32_t vf[4], vg[4];
      const int chunk = 4 * nq + (lane >> 3);
      ldsm_x4_t(vf, vbase + tok0 * kRowB + ((chunk ^ (tok0 & 7)) << 4));
      ldsm_x4_t(vg, vbase + tok1 * kRowB + ((chunk ^ (tok1 & 7)) << 4));
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float* oo = o[4 * nq + e];
        oo[0] *= corr;
        oo[1] *= corr;
        mma16816_top(o[4 * nq + e], pa0, pa2, vf[e], vg[e]);
        if (RLA) mma16816_top(o2[RLA ? 4 * nq + e : 0], wa0, wa2, vf[e], vg[e]);
      }
    }
    __syncthreads();
    slot = (slot + 1) % kRingC;

    if (++cur_sub >= stages_in(seg)) {
      // ---- end of segment: merge the warps' states per head
      float lq = l_run;
      lq += __shfl_xor_sync(0xffffffffu, lq, 1);
      lq += __shfl_xor_sync(0xffffffffu, lq, 2);
      if (hvalid) {
        float* mw = mg + ((size_t)hrow * kDecWarps + warp) * (D + 2);
        if ((lane & 3) == 0) {
          mw[0] = m_run;
          mw[1] = lq;
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          mw[2 + 8 * nt + 2 * (lane & 3)] = o[nt][0];
          mw[2 + 8 * nt + 2 * (lane & 3) + 1] = o[nt][1];
        }
      }
      __syncthreads();
      for (int x = tid; x < g * D; x += kDecThreads) {
        const int hh = x / D, c = x % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, mg[((size_t)hh * kDecWarps + w) * (D + 2)]);
        float L = 0.f, A = 0.f;
        if (M != -INFINITY) {
#pragma unroll
          for (int w = 0; w < kDecWarps; ++w) {
            const float* mw = mg + ((size_t)hh * kDecWarps + w) * (D + 2);
            if (mw[0] == -INFINITY) continue;
            const float f = fast_exp2(mw[0] - M);
            L = fmaf(mw[1], f, L);
            A = fmaf(mw[2 + c], f, A);
          }
        }
        float* out = partc + (((size_t)b * Hq + kh * g + hh) * nsegC + sseg) * (D + 2);
        if (c == 0) {
          out[0] = M;
          out[1] = L;
        }
        out[2 + c] = A;
      }
      __syncthreads();
      if (RLA) {
        // the residual linear sums add without a maximum: sum the warps'
        if (hvalid) {
          float* mw = mg + ((size_t)hrow * kDecWarps + warp) * (D + 2);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            mw[8 * nt + 2 * (lane & 3)] = o2[RLA ? nt : 0][0];
            mw[8 * nt + 2 * (lane & 3) + 1] = o2[RLA ? nt : 0][1];
          }
        }
        __syncthreads();
        for (int x = tid; x < g * D; x += kDecThreads) {
          const int hh = x / D, c = x % D;
          float A = 0.f;
#pragma unroll
          for (int w = 0; w < kDecWarps; ++w) A += mg[((size_t)hh * kDecWarps + w) * (D + 2) + c];
          partr[(((size_t)b * Hq + kh * g + hh) * nsegC + sseg) * D + c] = A;
        }
        __syncthreads();
      }
      cur_sub = 0;
      ++cur_seg_k;
    }
  }
  cp_async_wait<0>();
}

// ---- A'. statistics pass on the tensor cores (bf16 statistics) ------------
// The same outputs as decode_stats_kernel for bf16 kmean, kvar and value
// means.  A stage is 64 blocks of the three arrays, staged by cp.async
// (16-byte chunks of row r at chunk ^ (r & 7), as the exact pass stages K and
// V) into a ring (with the zero-order tail: four slots, three stages of
// 48 KB in flight while one is reduced; without it: two CTAs per SM with two
// slots each); a segment is two stages (128 blocks, the segments of
// decode_stats_kernel).  Warp w takes blocks [8w, 8w + 8) of a stage.  The dot
// products are mma.sync m16n8k16 contractions with the group's G <= 8 query
// heads as the MMA rows and the warp's 8 blocks as the columns:
// s log2e q·k̄_j (q and k̄ in bf16: exact products), and ½ s² Σ_c q_c² var_jc
// with ½ s² q² split into two bf16 terms (hi + lo: q² of a bf16 q has 16
// significant bits, so the split is exact).  The zero-order term of every
// block enters the warp's online softmax per head, its value-mean product
// P·v̄ on the tensor cores again (P in bf16, as the exact pass rounds its P;
// the warp's 8 blocks fill the MMA's first 8 k rows, the other 8 carry P = 0).
// At the end of a segment the warps' states are merged into one partial
// state per head as in decode_stats_kernel.
constexpr int kStageBlocksM = 64;
constexpr int kSegM = (kStageBlocksA * kSegA) / kStageBlocksM;   // stages per segment (2)
// ring slots and CTAs per SM: with the zero-order tail (three arrays and the
// P·v̄ accumulators) one CTA per SM with four slots; without it (two arrays)
// two CTAs per SM with two slots each (measured: 0.155 against 0.162 ms for
// the residual-linear decode step; the zero-order variant spills at two per
// SM and is slower)
template <bool ZT>
constexpr int ring_m() { return ZT ? 4 : 2; }
template <bool ZT>
constexpr int ctas_m() { return ZT ? 1 : 2; }

template <int D, bool ZT>
__global__ void __launch_bounds__(kDecThreads, ctas_m<ZT>())
decode_stats_mma_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ kmean,
                        const __nv_bfloat16* __restrict__ kvar, const __nv_bfloat16* __restrict__ vmean, int Hq,
                        int Hkv, int nb, int blk, float scale, int nsegA, int npairs, float* __restrict__ scores,
                        float* __restrict__ parta) {
  constexpr int CH = D / 8;                         // 16-byte chunks per bf16 row
  constexpr int NT = D / 8;                         // n-tiles of 8 channels
  constexpr int KS = D / 16;                        // k steps of 16 channels
  constexpr uint32_t kRowB = D * 2;
  constexpr uint32_t kArrB = kStageBlocksM * kRowB;
  constexpr int NARR = ZT ? 3 : 2;
  constexpr uint32_t kStageB = NARR * kArrB;
  constexpr int kRing = ring_m<ZT>();
  extern __shared__ __align__(16) uint8_t dsm[];
  const int g = Hq / Hkv;
  float* mg = reinterpret_cast<float*>(dsm);                         // [8 warps][g][D + 2] merge
  uint8_t* ring = dsm + ((sizeof(float) * kDecWarps * g * (D + 2) + 127) & ~(size_t)127);
  const uint32_t ring_s = (uint32_t)__cvta_generic_to_shared(ring);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int total_segs = npairs * nsegA;
  const float scale2 = scale * kLog2e;
  const float bias2 = log2f((float)blk);
  const int hrow = lane >> 2;                       // MMA row of this thread = query head
  const bool hvalid = hrow < g;
  const int nstage_pair = (nb + kStageBlocksM - 1) / kStageBlocksM;

  auto seg_of = [&](int k) { return (int)blockIdx.x + k * (int)gridDim.x; };
  auto stages_in = [&](int seg) { return min(kSegM, nstage_pair - (seg % nsegA) * kSegM); };
  // stage `sub` of segment `seg` into ring slot `slot`; rows past the pair's
  // last block are zero-filled
  auto issue = [&](int seg, int sub, int slot) {
    const int pair = seg / nsegA, j0 = ((seg % nsegA) * kSegM + sub) * kStageBlocksM;
    const int nrow = min(kStageBlocksM, nb - j0);
    const size_t base = ((size_t)pair * nb + j0) * D;
    uint8_t* dst = ring + slot * kStageB;
    for (int o = tid; o < kStageBlocksM * CH; o += kDecThreads) {
      const int r = o / CH, c = o % CH;
      const uint32_t sw = r * kRowB + ((c ^ (r & 7)) << 4);
      const size_t so = base + (size_t)(r < nrow ? r : 0) * D + 8 * c;
      const uint32_t nbytes = r < nrow ? 16u : 0u;
      cp_async16z(dst + sw, kmean + so, nbytes);
      cp_async16z(dst + kArrB + sw, kvar + so, nbytes);
      if (ZT) cp_async16z(dst + 2 * kArrB + sw, vmean + so, nbytes);
    }
  };
  if (seg_of(0) >= total_segs) return;
  int pf_k = 0, pf_sub = 0, pf_slot = 0;
  auto prefetch = [&]() {
    if (seg_of(pf_k) < total_segs) {
      issue(seg_of(pf_k), pf_sub, pf_slot);
      if (++pf_sub >= stages_in(seg_of(pf_k))) {
        pf_sub = 0;
        ++pf_k;
      }
    }
    cp_async_commit();
    pf_slot = (pf_slot + 1) % kRing;
  };
  for (int r = 0; r < kRing - 1; ++r) prefetch();

  uint32_t qa0[KS], qa2[KS];                  // q (rows = heads)
  uint32_t wh0[KS], wh2[KS], wl0[KS], wl2[KS];   // ½ s² q², hi and lo bf16 parts
  float m_run = -INFINITY, l_run = 0.f;       // the warp's zero-order state of head hrow
  float o[ZT ? NT : 1][2];
  int cur_pair = -1, cur_k = 0, cur_sub = 0, slot = 0;
  while (seg_of(cur_k) < total_segs) {
    const int seg = seg_of(cur_k);
    const int pair = seg / nsegA, sseg = seg % nsegA;
    const int b = pair / Hkv, kh = pair % Hkv;
    const int j0 = (sseg * kSegM + cur_sub) * kStageBlocksM;
    if (pair != cur_pair) {
      const __nv_bfloat16* qrow = q + ((size_t)b * Hq + kh * g + (hvalid ? hrow : 0)) * D;
#pragma unroll
      for (int kk = 0; kk < KS; ++kk) {
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int c0 = 16 * kk + 8 * half + 2 * (lane & 3);
          const uint32_t raw = *reinterpret_cast<const uint32_t*>(qrow + c0);
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw));
          const float w0 = 0.5f * scale * scale * f.x * f.x, w1 = 0.5f * scale * scale * f.y * f.y;
          const __nv_bfloat162 hi = __floats2bfloat162_rn(w0, w1);
          const float2 hf = __bfloat1622float2(hi);
          const uint32_t hiu = *reinterpret_cast<const uint32_t*>(&hi);
          const uint32_t lou = pack2bf16(w0 - hf.x, w1 - hf.y);
          if (half == 0) {
            qa0[kk] = hvalid ? raw : 0u;
            wh0[kk] = hvalid ? hiu : 0u;
            wl0[kk] = hvalid ? lou : 0u;
          } else {
            qa2[kk] = hvalid ? raw : 0u;
            wh2[kk] = hvalid ? hiu : 0u;
            wl2[kk] = hvalid ? lou : 0u;
          }
        }
      }
      cur_pair = pair;
    }
    if (ZT && cur_sub == 0) {
      m_run = -INFINITY;
      l_run = 0.f;
#pragma unroll
      for (int nt = 0; nt < (ZT ? NT : 1); ++nt) o[nt][0] = o[nt][1] = 0.f;
    }
    prefetch();
    cp_async_wait<kRing - 1>();
    __syncthreads();

    const uint32_t kbase = ring_s + slot * kStageB, vbase = kbase + 2 * kArrB;
    const int nrow = min(kStageBlocksM, nb - j0);
    const int tb = 8 * warp;
    const int r0 = tb + (lane & 7);             // the row this lane addresses
    // four independent accumulator chains (even / odd k steps; hi / lo of ½ s² q²)
    float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};   // q·k̄
    float ta[4] = {0.f, 0.f, 0.f, 0.f}, tb4[4] = {0.f, 0.f, 0.f, 0.f};  // ½ s² Σ q² var
#pragma unroll
    for (int kp = 0; kp < KS / 2; ++kp) {
      uint32_t kf[4], vf[4];
      const int chunk = 4 * kp + (lane >> 3);
      ldsm_x4(kf, kbase + r0 * kRowB + ((chunk ^ (r0 & 7)) << 4));
      ldsm_x4(vf, kbase + kArrB + r0 * kRowB + ((chunk ^ (r0 & 7)) << 4));
      mma16816_full(sa, qa0[2 * kp], qa2[2 * kp], kf[0], kf[1]);
      mma16816_full(sb, qa0[2 * kp + 1], qa2[2 * kp + 1], kf[2], kf[3]);
      mma16816_full(ta, wh0[2 * kp], wh2[2 * kp], vf[0], vf[1]);
      mma16816_full(tb4, wh0[2 * kp + 1], wh2[2 * kp + 1], vf[2], vf[3]);
      mma16816_full(ta, wl0[2 * kp], wl2[2 * kp], vf[0], vf[1]);
      mma16816_full(tb4, wl0[2 * kp + 1], wl2[2 * kp + 1], vf[2], vf[3]);
    }
    // the lane's two (head hrow, block) values: blocks tj, tj + 1
    const int tj = tb + 2 * (lane & 3);
    float x[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const bool live = hvalid && tj + e < nrow;
      const float d1 = (sa[e] + sb[e]) * scale2;   // s log2e q·k̄
      const float d2 = ta[e] + tb4[e];             // ½ s² Σ q² var
      // group score of the block, ln Σ_h e^{s q_h·k̄}(1 + d2_h) (the logsumexp
      // of the heads' log scores), in log2 units over the lanes 4 apart
      const float a = live ? d1 : -INFINITY;
      float mx = a;
#pragma unroll
      for (int o2 = 4; o2 < 32; o2 <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o2));
      float se = live ? fast_exp2(a - mx) * (1.0f + d2) : 0.f;
#pragma unroll
      for (int o2 = 4; o2 < 32; o2 <<= 1) se += __shfl_xor_sync(0xffffffffu, se, o2);
      if (hrow == 0 && tj + e < nrow) scores[(size_t)pair * nb + j0 + tj + e] = (mx + __log2f(se)) * kLn2;
      x[e] = live ? d1 + bias2 : -INFINITY;   // log2 weight of the block's pseudo-key
    }
    if (ZT) {
      // the warp's 8 blocks of head hrow: max over the row's four lanes
      float tmax = fmaxf(x[0], x[1]);
      tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
      tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 2));
      const float m_new = fmaxf(m_run, tmax);
      const float corr = m_run == -INFINITY ? 0.f : fast_exp2(m_run - m_new);
      const float p0 = x[0] != -INFINITY ? fast_exp2(x[0] - m_new) : 0.f;
      const float p1 = x[1] != -INFINITY ? fast_exp2(x[1] - m_new) : 0.f;
      l_run = l_run * corr + (p0 + p1);
      m_run = m_new;
      const uint32_t pa0 = pack2bf16(p0, p1);
#pragma unroll
      for (int nq = 0; nq < NT / 4; ++nq) {
        uint32_t vv[4];
        const int chunk = 4 * nq + (lane >> 3);
        ldsm_x4_t(vv, vbase + r0 * kRowB + ((chunk ^ (r0 & 7)) << 4));
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float* oo = o[ZT ? 4 * nq + e : 0];
          oo[0] *= corr;
          oo[1] *= corr;
          // k rows 8-15 carry P = 0 (their B operand repeats rows 0-7)
          mma16816_top(o[ZT ? 4 * nq + e : 0], pa0, 0u, vv[e], vv[e]);
        }
      }
    }
    slot = (slot + 1) % kRing;
    const bool seg_end = ++cur_sub >= stages_in(seg);
    if (ZT && seg_end) {
      // the warp's state of head hrow for this segment, then the merge
      float lq = l_run;
      lq += __shfl_xor_sync(0xffffffffu, lq, 1);
      lq += __shfl_xor_sync(0xffffffffu, lq, 2);
      if (hvalid) {
        float* mw = mg + ((size_t)warp * g + hrow) * (D + 2);
        if ((lane & 3) == 0) {
          mw[0] = m_run;
          mw[1] = lq;
        }
#pragma unroll
        for (int nt = 0; nt < (ZT ? NT : 1); ++nt) {
          mw[2 + 8 * nt + 2 * (lane & 3)] = o[nt][0];
          mw[2 + 8 * nt + 2 * (lane & 3) + 1] = o[nt][1];
        }
      }
      __syncthreads();
      for (int xi = tid; xi < g * D; xi += kDecThreads) {
        const int hh = xi / D, c = xi % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, mg[((size_t)w * g + hh) * (D + 2)]);
        float Lm = 0.f, A = 0.f;
        if (M != -INFINITY) {
#pragma unroll
          for (int w = 0; w < kDecWarps; ++w) {
            const float* mw = mg + ((size_t)w * g + hh) * (D + 2);
            if (mw[0] == -INFINITY) continue;
            const float f = fast_exp2(mw[0] - M);
            Lm = fmaf(mw[1], f, Lm);
            A = fmaf(mw[2 + c], f, A);
          }
        }
        float* out = parta + (((size_t)b * Hq + kh * g + hh) * nsegA + sseg) * (D + 2);
        if (c == 0) {
          out[0] = M;
          out[1] = Lm;
        }
        out[2 + c] = A;
      }
    }
    __syncthreads();   // the slot is restaged by a later prefetch; the merge rows are free
    if (seg_end) {
      cur_sub = 0;
      ++cur_k;
    }
  }
  cp_async_wait<0>();
}

// ---- D. merge ------------------------------------------------------------
// One CTA of D threads per (sequence, KV head), thread = channel, for the
// group's G query heads.  It merges the statistics pass's partial states (the
// zero-order term of every block) with the exact pass's (the selected blocks
// token by token) under their common maximum, after subtracting the
// zero-order term of each selected block (SPLA §2.2's subtraction applied to
// PISA's tail: the statistics pass cannot know the selection), so that the
// tail holds the unselected blocks only.  The subtraction cannot go below
// zero: for every block Σ_n e^{x_n} ≥ B e^{mean x}, and the statistics
// states' maximum M_A bounds every block's zero-order logit, so no weight
// 2^{x_j − M_A} exceeds 1.
// Everything but the exact pass's states is formed before the PDL wait: the
// statistics states merged per head under M_A, the selected blocks' weights
// (q·k̄_j, a warp per block) subtracted there, and with the residual linear
// tail φ(q)ᵀ S_all.  The exact pass leaves room for one such CTA per SM, so
// with at most one CTA per SM this work overlaps the pass and after it only
// the exact states' merge remains.  States are merged a chunk at a time
// (online, as the passes merge tokens): their (max, sum) pairs staged in
// shared memory, the maxima and weights formed by a warp per head, and each
// thread's channel values loaded in batches of 32 / G so that the loads of
// a batch are in flight together.
constexpr float kRmsEps = 1e-6f;     // RMSNorm of SPLA's residual linear output
constexpr int kSelChunk = 64;        // selected blocks whose weights are staged at once
constexpr int kStChunk = 128;        // (head, state) pairs staged at once

__device__ __forceinline__ float ld_stat(const float* p) { return __ldg(p); }
__device__ __forceinline__ float ld_stat(const __nv_bfloat16* p) { return __bfloat162float(__ldg(p)); }

// shared memory of decode_combine_kernel (floats)
__host__ __device__ constexpr int combine_smem_floats(int g, int D, bool rla) {
  return g * D + (rla ? g * D : 0) + 2 * kStChunk + g * kSelChunk + kSelChunk + 3 * g + g * (D / 32);
}

// TS, kmean, vrow, vmul: the statistics as the statistics pass read them
// (vmul turns a row of vrow into the block's value mean)
template <int D, int G, typename TS>
__global__ void __launch_bounds__(D, 640 / D)
decode_combine_kernel(const float* __restrict__ parta, int nsegA, const float* __restrict__ partc, int nsegC,
                      int use_tail, const float* __restrict__ partr, const __nv_bfloat16* __restrict__ q,
                      const TS* __restrict__ kmean, const TS* __restrict__ vrow, float vmul,
                      const float* __restrict__ sexp, const int32_t* __restrict__ idx, int topk, int nb, int blk,
                      float scale, int Hkv, __nv_bfloat16* __restrict__ O) {
  // Everything up to the pdl_wait() below comes from the earlier launches of
  // the step (statistics pass, top-k), which had completed before the exact
  // pass read the selection; only the exact pass's partial states (partc,
  // partr) are read after it.
  constexpr int kW = D / 32;
  constexpr int kB = 32 / G;                                   // states per load batch
  extern __shared__ __align__(16) float csm[];
  const int Hq = Hkv * G;
  const int pair = blockIdx.x, b = pair / Hkv;
  const size_t row0 = (size_t)b * Hq + (size_t)(pair % Hkv) * G;   // the group's heads: rows row0 .. row0 + G - 1
  const int c = threadIdx.x, lane = c & 31, warp = c >> 5;
  const int na = use_tail ? nsegA : 0;
  const int nsel = (use_tail && nsegC > 0) ? topk : 0;
  const bool rla = partr != nullptr;
  float* qs = csm;                                             // [G][D] s log2e q
  float* fq = qs + G * D;                                      // [G][D] φ(q) in bf16 (residual linear)
  float* sm = fq + (rla ? G * D : 0);                          // [kStChunk] state maxima, then weights
  float* sl = sm + kStChunk;                                   // [kStChunk] state sums
  float* wsel = sl + kStChunk;                                 // [G][kSelChunk] weights 2^{x_j − M_A}
  int* jsel = reinterpret_cast<int*>(wsel + G * kSelChunk);    // [kSelChunk] block indices
  float* hM = reinterpret_cast<float*>(jsel + kSelChunk);      // [G] running maximum per head
  float* hL = hM + G;                                          // [G] running sum per head
  float* hS = hL + G;                                          // [G] rescale of the last chunk
  float* red = hS + G;                                         // [G][kW] RMS partial sums
  const float scale2 = scale * kLog2e, bias2 = log2f((float)blk);
  for (int x = c; x < G * D; x += D) {
    const float qv = __bfloat162float(q[row0 * D + x]);
    qs[x] = scale2 * qv;
    // φ(q) rounded to bf16 as in the exact pass's operand, so that the two
    // terms of the residual's difference use the same feature values
    if (rla) fq[x] = __bfloat162float(__float2bfloat16_rn(phi_exp(qv)));
  }
  if (c < G) {
    hM[c] = -INFINITY;
    hL[c] = 0.f;
  }
  __syncthreads();   // qs, fq, hM, hL
  float A[G];
#pragma unroll
  for (int hh = 0; hh < G; ++hh) A[hh] = 0.f;

  // merge states x ∈ [0, nst) of the group's heads (rows of D + 2 floats at
  // base + ((row0 + hh) nst + x)(D + 2)) into (hM, hL) and A
  auto merge_states = [&](const float* base, int nst) {
    constexpr int per = kStChunk / G;
    for (int x0 = 0; x0 < nst; x0 += per) {
      const int n = min(per, nst - x0);
      for (int z = c; z < G * n; z += D) {
        const float* r = base + ((row0 + z / n) * nst + x0 + z % n) * (D + 2);
        sm[z] = r[0];
        sl[z] = r[1];
      }
      __syncthreads();
      for (int hh = warp; hh < G; hh += kW) {
        float cm = -INFINITY;
        for (int x = lane; x < n; x += 32) cm = fmaxf(cm, sm[hh * n + x]);
        cm = warp_max(cm);
        const float mo = hM[hh], mn = fmaxf(mo, cm);
        float ls = 0.f;
        for (int x = lane; x < n; x += 32) {
          const float m = sm[hh * n + x];
          const float w = m == -INFINITY ? 0.f : fast_exp2(m - mn);
          sm[hh * n + x] = w;
          ls = fmaf(sl[hh * n + x], w, ls);
        }
        ls = warp_sum(ls);
        if (lane == 0) {
          const float so = mo == -INFINITY ? 0.f : fast_exp2(mo - mn);
          hS[hh] = so;
          hL[hh] = fmaf(hL[hh], so, ls);
          hM[hh] = mn;
        }
      }
      __syncthreads();
#pragma unroll
      for (int hh = 0; hh < G; ++hh) A[hh] *= hS[hh];
      for (int x = 0; x < n; x += kB) {
        float v[G][kB];
#pragma unroll
        for (int hh = 0; hh < G; ++hh)
#pragma unroll
          for (int u = 0; u < kB; ++u)
            v[hh][u] = x + u < n ? base[((row0 + hh) * nst + x0 + x + u) * (D + 2) + 2 + c] : 0.f;
#pragma unroll
        for (int hh = 0; hh < G; ++hh)
#pragma unroll
          for (int u = 0; u < kB; ++u)
            if (x + u < n) A[hh] = fmaf(v[hh][u], sm[hh * n + x + u], A[hh]);
      }
      __syncthreads();   // sm, sl are restaged by the next chunk
    }
  };

  // the statistics pass's states (zero-order terms of every block) under M_A
  merge_states(parta, na);

  // subtract the zero-order term of each selected block (weight <= 1)
  float lsub[G];
#pragma unroll
  for (int hh = 0; hh < G; ++hh) lsub[hh] = 0.f;
  for (int s0 = 0; s0 < nsel; s0 += kSelChunk) {
    const int n = min(kSelChunk, nsel - s0);
    if (c < n) jsel[c] = __ldg(idx + (size_t)pair * topk + s0 + c);
    __syncthreads();
    // s log2e q_h·k̄_j + log2 B − M_A(h): a warp per block, eight blocks in flight
    for (int u0 = warp * 8; u0 < n; u0 += kW * 8) {
      float kk[8][D / 32];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const TS* kr = kmean + ((size_t)pair * nb + jsel[min(u0 + u, n - 1)]) * D;
#pragma unroll
        for (int e = 0; e < D / 32; ++e) kk[u][e] = ld_stat(kr + lane + 32 * e);
      }
#pragma unroll
      for (int hh = 0; hh < G; ++hh) {
        const float ma = hM[hh];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          float d = 0.f;
#pragma unroll
          for (int e = 0; e < D / 32; ++e) d = fmaf(qs[hh * D + lane + 32 * e], kk[u][e], d);
          d = warp_sum(d);
          if (lane == 0 && u0 + u < n)
            wsel[hh * kSelChunk + u0 + u] = ma == -INFINITY ? 0.f : fast_exp2(d + bias2 - ma);
        }
      }
    }
    __syncthreads();
    for (int u0 = 0; u0 < n; u0 += 16) {
      float v[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) v[u] = ld_stat(vrow + ((size_t)pair * nb + jsel[min(u0 + u, n - 1)]) * D + c);
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        if (u0 + u < n) {
#pragma unroll
          for (int hh = 0; hh < G; ++hh) {
            const float w = wsel[hh * kSelChunk + u0 + u];
            lsub[hh] += w;
            A[hh] = fmaf(-w * vmul, v[u], A[hh]);
          }
        }
      }
    }
    __syncthreads();   // jsel and wsel are restaged by the next chunk
  }
  if (c == 0 && nsel > 0) {
#pragma unroll
    for (int hh = 0; hh < G; ++hh) hL[hh] -= lsub[hh];
  }

  // SPLA's residual: φ(q)ᵀ S_all (column c) for each head of the group
  float res[G];
#pragma unroll
  for (int hh = 0; hh < G; ++hh) res[hh] = 0.f;
  if (rla) {
    const float* sa = sexp + (size_t)pair * D * D;
#pragma unroll 16
    for (int r = 0; r < D; ++r) {
      const float sv = __ldg(sa + (size_t)r * D + c);
#pragma unroll
      for (int hh = 0; hh < G; ++hh) res[hh] = fmaf(fq[hh * D + r], sv, res[hh]);
    }
  }

  pdl_wait();   // the exact pass's partial states from here on
  merge_states(partc, nsegC);   // its first barrier orders thread 0's update of hL
  if (rla) {
    // minus the exact segments' Σ (φ(q)·φ(k_n)) v_n, then RMSNorm over the
    // D channels of each head
    for (int x = 0; x < nsegC; x += kB) {
      float v[G][kB];
#pragma unroll
      for (int hh = 0; hh < G; ++hh)
#pragma unroll
        for (int u = 0; u < kB; ++u) v[hh][u] = x + u < nsegC ? partr[((row0 + hh) * nsegC + x + u) * D + c] : 0.f;
#pragma unroll
      for (int hh = 0; hh < G; ++hh)
#pragma unroll
        for (int u = 0; u < kB; ++u) res[hh] -= v[hh][u];
    }
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
      const float sq = warp_sum(res[hh] * res[hh]);
      if (lane == 0) red[hh * kW + warp] = sq;
    }
    __syncthreads();
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
      float tot = 0.f;
#pragma unroll
      for (int w = 0; w < kW; ++w) tot += red[hh * kW + w];
      res[hh] *= rsqrtf(tot / D + kRmsEps);
    }
  }
  __syncthreads();   // hL
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    const float L = hL[hh];
    const float o_s = L > 0.f ? A[hh] / L : 0.f;
    O[(row0 + hh) * D + c] = __float2bfloat16_rn(o_s + res[hh]);
  }
}

int sm_count() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

// The statistics the decode reads: float32 kmean, kvar, vsum, or (when
// kmean is NULL) their bf16 copies kmean_bf16, kvar_bf16, vmean_bf16.
template <typename TS>
struct DecodeStats {
  const TS *kmean, *kvar, *vrow;
  float vmul;   // vrow row -> block value mean
};

template <int D, typename TS>
sa_status launch_decode(const void* q, const void* Kc, const void* Vc, const sa_decode_shape& s,
                        const sa_block_stats& st, const DecodeStats<TS>& ds, int topk, float scale,
                        sa_tail_mode tail, int32_t* idx_out, float* scores_out, void* O, char* ws,
                        cudaStream_t stream) {
  const DecodeLayout L = decode_layout(s, topk);
  const int nb = s.N / s.block;
  const int npairs = s.B * s.Hkv;
  float* scores = scores_out ? scores_out : reinterpret_cast<float*>(ws + L.scores_off);
  int32_t* idx = idx_out ? idx_out : reinterpret_cast<int32_t*>(ws + L.idx_off);
  float* parta = reinterpret_cast<float*>(ws + L.parta_off);
  float* partc = reinterpret_cast<float*>(ws + L.partc_off);
  // residual linear tail: with every block selected U is empty and the
  // residual is zero by definition (the difference S_all − S_sel would only
  // hold rounding noise, which the RMS norm would blow up to unit size)
  const bool rla = tail == SA_TAIL_RESIDUAL_LINEAR;
  float* partr = rla ? reinterpret_cast<float*>(ws + L.partr_off) : nullptr;
  const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(q);
  const int sms = sm_count();
  bool topk_done = false;   // the tensor-core statistics pass may select the blocks itself

  // A
  {
    const int g = s.Hq / s.Hkv;
    constexpr int RING = ring_a<TS>();
    const size_t smemA = sizeof(float) * (kThrA / 32) * g * (D + 2) + 16 * RING +
                         (size_t)RING * 3 * kStageBlocksA * D * sizeof(TS);
    const long segsA = (long)npairs * L.nsegA;
    const int gridA = (int)(segsA < 2 * sms ? segsA : 2 * sms);
    sa_status r0 = SA_OK;
    auto run = [&](auto kern) {
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smemA) != cudaSuccess) {
        r0 = launch_status("cudaFuncSetAttribute(decode_stats_kernel)");
        return;
      }
      kern<<<gridA, kThrA, smemA, stream>>>(qb, ds.kmean, ds.kvar, ds.vrow, ds.vmul, s.Hq, s.Hkv, nb, s.block,
                                            scale, L.nsegA, npairs, scores, parta);
      r0 = launch_status("decode_stats_kernel");
    };
    const bool zt = tail == SA_TAIL_ZERO_ORDER;
    if constexpr (sizeof(TS) == 2) {
      if (D == 128 && g <= 16) {
        // bf16 statistics, d = 128: the tcgen05 statistics pass (decode_tc.cu)
        r0 = decode_stats_tc(qb, ds.kmean, ds.kvar, ds.vrow, s.B, s.Hq, s.Hkv, nb, s.block, scale, L.nsegA, zt,
                             sms, scores, parta, topk, idx, &topk_done, stream);
      } else {
        // bf16 statistics otherwise: the mma.sync statistics pass (one or two CTAs per SM)
        const size_t smemM = ((sizeof(float) * kDecWarps * g * (D + 2) + 127) & ~(size_t)127) +
                             (size_t)(zt ? ring_m<true>() : ring_m<false>()) * (zt ? 3 : 2) * kStageBlocksM * D * 2;
        const int per_sm = zt ? ctas_m<true>() : ctas_m<false>();
        const int gridM = (int)(segsA < per_sm * sms ? segsA : per_sm * sms);
        auto kern = zt ? decode_stats_mma_kernel<D, true> : decode_stats_mma_kernel<D, false>;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smemM) != cudaSuccess)
          return launch_status("cudaFuncSetAttribute(decode_stats_mma_kernel)");
        kern<<<gridM, kDecThreads, smemM, stream>>>(qb, ds.kmean, ds.kvar, ds.vrow, s.Hq, s.Hkv, nb, s.block, scale,
                                                    L.nsegA, npairs, scores, parta);
        r0 = launch_status("decode_stats_mma_kernel");
      }
    } else if (g == 1) run(zt ? decode_stats_kernel<D, 1, true, TS> : decode_stats_kernel<D, 1, false, TS>);
    else if (g == 2) run(zt ? decode_stats_kernel<D, 2, true, TS> : decode_stats_kernel<D, 2, false, TS>);
    else if (g == 4) run(zt ? decode_stats_kernel<D, 4, true, TS> : decode_stats_kernel<D, 4, false, TS>);
    else run(zt ? decode_stats_kernel<D, 8, true, TS> : decode_stats_kernel<D, 8, false, TS>);
    if (r0 != SA_OK) return r0;
  }
  sa_status r = SA_OK;

  // B (unless the statistics pass selected the blocks already)
  if (topk > 0 && !topk_done) {
    {
      const cudaError_t le = launch_pdl(decode_topk_kernel, dim3(npairs), dim3(kDecThreads), 0, stream, scores, nb, topk, idx);
      if (le != cudaSuccess) return fail(SA_ERR_CUDA, std::string("decode_topk_kernel: ") + cudaGetErrorString(le));
    }
    r = launch_status("decode_topk_kernel");
    if (r != SA_OK) return r;
  }

  // C
  if (topk > 0) {
    const size_t smemC = sizeof(float) * exact_merge_floats(s.Hq / s.Hkv, D) +
                         sizeof(int) * kItabSegs * (kSegC * kStageTokC / 64) +
                         (size_t)kRingC * 2 * kStageTokC * D * 2;
    auto kern = rla ? decode_exact_kernel<D, true> : decode_exact_kernel<D, false>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smemC) != cudaSuccess)
      return launch_status("cudaFuncSetAttribute(decode_exact_kernel)");
    const long segsC = (long)npairs * L.nsegC;   // < 2^31 for any supported shape
    const int gridC = (int)(segsC < sms ? segsC : sms);
    {
      const cudaError_t le = launch_pdl(kern, dim3(gridC), dim3(kDecThreads), smemC, stream,
        qb, static_cast<const __nv_bfloat16*>(Kc), static_cast<const __nv_bfloat16*>(Vc), s.Hq, s.Hkv, s.N,
        s.block, idx, topk, scale, L.nsegC, npairs, partc, partr);
      if (le != cudaSuccess) return fail(SA_ERR_CUDA, std::string("decode_exact_kernel: ") + cudaGetErrorString(le));
    }
    r = launch_status("decode_exact_kernel");
    if (r != SA_OK) return r;
  }

  // D
  {
    const int use_tail = tail == SA_TAIL_ZERO_ORDER;
    const int nsc = topk > 0 ? L.nsegC : 0;
    const float* pr = topk < nb ? partr : nullptr;
    const int g = s.Hq / s.Hkv;
    const size_t smemD = sizeof(float) * combine_smem_floats(g, D, pr != nullptr);
    auto kern = g == 1 ? decode_combine_kernel<D, 1, TS> : g == 2 ? decode_combine_kernel<D, 2, TS>
              : g == 4 ? decode_combine_kernel<D, 4, TS> : decode_combine_kernel<D, 8, TS>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smemD) != cudaSuccess)
      return launch_status("cudaFuncSetAttribute(decode_combine_kernel)");
    {
      const cudaError_t le = launch_pdl(kern, dim3(npairs), dim3(D), smemD, stream, parta, L.nsegA, partc, nsc,
        use_tail, pr, qb, ds.kmean, ds.vrow, ds.vmul, static_cast<const float*>(st.sexp), idx, topk, nb, s.block,
        scale, s.Hkv, static_cast<__nv_bfloat16*>(O));
      if (le != cudaSuccess) return fail(SA_ERR_CUDA, std::string("decode_combine_kernel: ") + cudaGetErrorString(le));
    }
  }
  return launch_status("decode_combine_kernel");
}

sa_status check_decode_shape(const sa_decode_shape& s, int topk) {
  if (s.B < 0 || s.Hq <= 0 || s.Hkv <= 0 || s.N < 0)
    return fail(SA_ERR_INVALID_ARG, "sa_decode_fwd: negative or zero size");
  if (s.Hq % s.Hkv) return fail(SA_ERR_INVALID_ARG, "sa_decode_fwd: Hq must be a multiple of Hkv");
  if (s.Hq / s.Hkv > kMaxGroup || (kMaxGroup % (s.Hq / s.Hkv)))
    return fail(SA_ERR_UNSUPPORTED, "sa_decode_fwd: the GQA group (Hq / Hkv) must be 1, 2, 4 or 8");
  if (s.d != 64 && s.d != 128) return fail(SA_ERR_UNSUPPORTED, "sa_decode_fwd: d must be 64 or 128");
  if (s.block != 64 && s.block != 128) return fail(SA_ERR_UNSUPPORTED, "sa_decode_fwd: block must be 64 or 128");
  if (s.N % s.block) return fail(SA_ERR_INVALID_ARG, "sa_decode_fwd: N must be a multiple of block");
  const int nb = s.N / s.block;
  if (nb > kMaxRouteBlocks) return fail(SA_ERR_UNSUPPORTED, "sa_decode_fwd: at most 4096 blocks per sequence");
  if (topk < 0 || topk > nb) return fail(SA_ERR_INVALID_ARG, "sa_decode_fwd: topk must be in [0, N/block]");
  return SA_OK;
}

}  // namespace
}  // namespace sa

namespace sa {
uint32_t decode_error_take() {
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_decode_error, sizeof(v)) != cudaSuccess ||
      cudaMemcpyToSymbol(g_decode_error, &zero, sizeof(zero)) != cudaSuccess)
    return 0u;
  return v;
}
}  // namespace sa

extern "C" size_t sa_decode_workspace_size(sa_decode_shape shape, int32_t topk) {
  using namespace sa;
  if (check_decode_shape(shape, topk) != SA_OK) return 0;
  return decode_layout(shape, topk).total;
}

extern "C" sa_status sa_decode_fwd(const void* q, const void* Kcache, const void* Vcache,
                                   sa_dtype dtype, sa_decode_shape shape,
                                   const sa_block_stats* stats, int32_t topk, float scale,
                                   sa_tail_mode tail, int32_t* block_idx_out, float* scores_out,
                                   void* O, void* workspace, size_t workspace_bytes, void* stream) {
  using namespace sa;
  sa_status r = check_decode_shape(shape, topk);
  if (r != SA_OK) return r;
  if (dtype != SA_BF16) return fail(SA_ERR_UNSUPPORTED, "sa_decode_fwd: bf16 caches only");
  if (tail != SA_TAIL_ZERO_ORDER && tail != SA_TAIL_DROP && tail != SA_TAIL_RESIDUAL_LINEAR)
    return fail(SA_ERR_UNSUPPORTED,
                "sa_decode_fwd: tail must be SA_TAIL_DROP, SA_TAIL_ZERO_ORDER or SA_TAIL_RESIDUAL_LINEAR");
  if (!q || !Kcache || !Vcache || !O || !stats)
    return fail(SA_ERR_INVALID_ARG, "sa_decode_fwd: q, caches, O and stats are required");
  const bool stats_bf16 = stats->kmean == nullptr;
  if (!stats_bf16 && (!stats->kvar || !stats->vsum))
    return fail(SA_ERR_INVALID_ARG, "sa_decode_fwd: float32 statistics need kmean, kvar and vsum");
  if (stats_bf16 && (!stats->kmean_bf16 || !stats->kvar_bf16 || (tail == SA_TAIL_ZERO_ORDER && !stats->vmean_bf16)))
    return fail(SA_ERR_INVALID_ARG,
                "sa_decode_fwd: without stats->kmean the bf16 statistics kmean_bf16, kvar_bf16 (and vmean_bf16 "
                "for SA_TAIL_ZERO_ORDER) are required");
  if (tail == SA_TAIL_RESIDUAL_LINEAR && !stats->sexp)
    return fail(SA_ERR_INVALID_ARG, "sa_decode_fwd: SA_TAIL_RESIDUAL_LINEAR needs stats->sexp");
  const void* ptrs[] = {q, Kcache, Vcache, O, stats->kmean, stats->kvar, stats->vsum, stats->sexp, block_idx_out,
                        scores_out, stats->kmean_bf16, stats->kvar_bf16, stats->vmean_bf16};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(SA_ERR_ALIGNMENT, "sa_decode_fwd: pointers must be 16-byte aligned");
  const size_t need = decode_layout(shape, topk).total;
  if (!workspace || workspace_bytes < need)
    return fail(SA_ERR_WORKSPACE, "sa_decode_fwd: workspace missing or smaller than sa_decode_workspace_size()");
  if (reinterpret_cast<uintptr_t>(workspace) & 255u)
    return fail(SA_ERR_ALIGNMENT, "sa_decode_fwd: workspace must be 256-byte aligned");
  if (shape.B == 0 || shape.N == 0) return SA_OK;
  cudaStream_t s = as_stream(stream);
  char* ws = static_cast<char*>(workspace);
  if (stats_bf16) {
    typedef __nv_bfloat16 bf;
    // vmean_bf16 may be NULL without the zero-order tail; the kernels then never read it
    const DecodeStats<bf> ds{reinterpret_cast<const bf*>(stats->kmean_bf16),
                             reinterpret_cast<const bf*>(stats->kvar_bf16),
                             reinterpret_cast<const bf*>(stats->vmean_bf16), 1.0f};
    if (shape.d == 128)
      return launch_decode<128, bf>(q, Kcache, Vcache, shape, *stats, ds, topk, scale, tail, block_idx_out,
                                    scores_out, O, ws, s);
    return launch_decode<64, bf>(q, Kcache, Vcache, shape, *stats, ds, topk, scale, tail, block_idx_out,
                                 scores_out, O, ws, s);
  }
  const DecodeStats<float> ds{stats->kmean, stats->kvar, stats->vsum, 1.0f / shape.block};
  if (shape.d == 128)
    return launch_decode<128, float>(q, Kcache, Vcache, shape, *stats, ds, topk, scale, tail, block_idx_out,
                                     scores_out, O, ws, s);
  return launch_decode<64, float>(q, Kcache, Vcache, shape, *stats, ds, topk, scale, tail, block_idx_out,
                                  scores_out, O, ws, s);
}

// ---- decode with library-owned scratch ---------------------------------------
// sa_decode_fwd_static runs the same kernels as sa_decode_fwd, with its
// scratch (route scores, selected indices, per-split partial states) in this
// file-scope device array instead of a caller workspace.  The array exists
// once per CUDA context that loads the library's module and stays allocated
// until that context is destroyed (for the primary context: process exit or
// cudaDeviceReset).  Host code must not hand `g_decode_scratch` itself to a
// kernel (on the host it names a shadow variable, not device memory); its
// device address is looked up with cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_decode_scratch[SA_DECODE_STATIC_SCRATCH_BYTES];

namespace {
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

struct CtxFns {
  CtxGetCurrentFn get_current = nullptr;
  CtxGetIdFn get_id = nullptr;
};

const CtxFns& ctx_fns() {
  static CtxFns f;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      f.get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      f.get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  return f;
}

// Unique id of the current context (cuCtxGetId: ids are never reused within
// a process, unlike context handles or device indices); 0 if none is current.
unsigned long long current_ctx_id() {
  const CtxFns& f = ctx_fns();
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!f.get_current || !f.get_id || f.get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  if (f.get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

std::mutex g_scratch_mu;
// (context id, device address of g_decode_scratch in that context)
std::vector<std::pair<unsigned long long, void*>> g_scratch_addr;

// Device address of g_decode_scratch in the current context.  The address
// belongs to the copy of the module loaded into one context, so it is cached
// per context id: a context created by cudaDeviceReset, or a caller's own
// context made current instead of the primary one, gets a lookup of its own.
// The lookup (cudaGetSymbolAddress) also initialises the primary context
// when none is current yet.
sa_status static_scratch(void** out) {
  using namespace sa;
  unsigned long long id = current_ctx_id();
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (id != 0)
    for (const auto& e : g_scratch_addr)
      if (e.first == id) {
        *out = e.second;
        return SA_OK;
      }
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
  if (e != cudaSuccess || p == nullptr)
    return fail(SA_ERR_CUDA, std::string("sa_decode_fwd_static: cudaGetSymbolAddress failed: ") +
                                 cudaGetErrorString(e));
  if (id == 0) id = current_ctx_id();   // the lookup made the primary context current
  if (id != 0) g_scratch_addr.emplace_back(id, p);
  *out = p;
  return SA_OK;
}
}  // namespace

extern "C" sa_status sa_decode_fwd_static(const void* q, const void* Kcache, const void* Vcache,
                                          sa_dtype dtype, sa_decode_shape shape,
                                          const sa_block_stats* stats, int32_t topk, float scale,
                                          sa_tail_mode tail, int32_t* block_idx_out,
                                          float* scores_out, void* O, void* stream) {
  using namespace sa;
  const size_t need = sa_decode_workspace_size(shape, topk);
  if (need > SA_DECODE_STATIC_SCRATCH_BYTES)
    return fail(SA_ERR_WORKSPACE, "sa_decode_fwd_static: this problem needs " + std::to_string(need) +
                                      " bytes of scratch; the library's static scratch holds " +
                                      std::to_string((size_t)SA_DECODE_STATIC_SCRATCH_BYTES) +
                                      " bytes (use sa_decode_fwd with a workspace)");
  void* scratch = nullptr;
  sa_status r = static_scratch(&scratch);
  if (r != SA_OK) return r;
  // every scratch entry the kernels read is written earlier in the same call,
  // so the contents left by a previous call need no clearing
  return sa_decode_fwd(q, Kcache, Vcache, dtype, shape, stats, topk, scale, tail, block_idx_out,
                       scores_out, O, scratch, SA_DECODE_STATIC_SCRATCH_BYTES, stream);
}

// far_kernels.cu -- sm_100a kernels of the fused "all-reduce + residual-add +
// RMSNorm (+FP8-e4m3)" epilogue.
//
// Per row t (fused_allreduce_rms_norm docstring on the
// vllm.models.common.ops.fused_allreduce_rms_norm page: the result is
// norm(all_reduce(h), residual) with fp32 accumulation):
//   y = sum_r p_r + residual          -> residual_out = round(y)
//   rinv = 1/sqrt(mean(y^2) + eps)
//   o = y * rinv * (gamma + weight_bias) -> norm_out = round(o)
//   static FP8 (FusedAddRMSNormStaticQuantPattern): q = e4m3(o / scale)
//   per-token FP8 (FusedAddRMSNormDynamicQuantPattern):
//       scale_t = max|o| / 448, q = e4m3(o / scale_t)
//
// The work is HBM-bound (about 8 flops per (W+3)*2 bytes): no tensor cores.
// A whole row stays in registers between its reduction and its scaling, so
// every byte crosses HBM once.  Four kernels, three of which share one row
// routine (finish_row), and a one-CTA helper:
//  - far_ring_kernel (prefill, many rows): persistent CTAs; one producer
//    thread streams each row's segments with TMA bulk copies into a ring of
//    shared-memory slots, the consumer warps fold them into registers; for
//    dynamic per-tensor FP8 it also runs both passes in one launch (rows
//    taken from a counter, a bounded wait until every row is done);
//  - far_prefill_kernel (fewer rows): one CTA per row (or 256/tpr rows per
//    CTA when a row has at most 32 packs), 16-byte vector loads issued
//    ahead of their use, warp-shuffle + shared-memory reductions;
//  - far_decode_kernel (a few long rows): one thread-block cluster per row,
//    each CTA a slice of the hidden dimension, the row's sum of squares
//    (and amax) combined through distributed shared memory;
//  - far_tensor_quant_kernel: the second pass of dynamic per-tensor FP8 in
//    its two-kernel form, codes from the stored new residual (no reduction);
//  - far_ws_zero_kernel: zeroes the per-tensor workspace header.
#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "far_internal.h"

namespace cg = cooperative_groups;

namespace far {
namespace {

// Shared-memory layout of the ring kernel: nslot "full" and nslot "empty"
// mbarriers (8 bytes each), a RingHeader, then from a 128-byte boundary
// gamma (H*2 bytes, loaded once per CTA) and the nslot slots.
struct RingHeader {
  float red[2][2][32];   // [row parity][0 = sum of squares, 1 = amax][warp]
  int slot_row[32];      // rows taken from a shared counter: the row (ordinal)
                         // whose first segment sits in the slot, -1: no more rows
  float slot_w[32];      // per-tensor second pass: that row's stored rinv (flag)
  int abort;             // set when any wait of the CTA gave up
  int producer_done;     // set by the producer when it stops issuing
  long long issued;      // bulk copies the producer issued
};

__host__ __device__ constexpr int ring_offset(int nslot) {
  return (16 * nslot + static_cast<int>(sizeof(RingHeader)) + 127) / 128 * 128;
}

// Which instantiation serves a pattern: the per-group and the per-tensor
// passes have kernels of their own, so that the other patterns' code carries
// none of their registers.
// kModeTensorNorm: per-tensor FP8 whose second pass forms the codes from the
// norm_out the first pass stores (its own instantiations, so that the other
// per-tensor forms carry none of that code)
constexpr int kModePlain = 0, kModeGroup = 1, kModeTensor = 2, kModeTensorNorm = 3;
__host__ __device__ constexpr bool is_tensor_mode(int mode) {
  return mode == kModeTensor || mode == kModeTensorNorm;
}
__host__ __device__ constexpr int mode_of(int pattern) {
  return pattern == kFp8Group ? kModeGroup
         : (pattern == kTensorAmax || pattern == kTensorQuant) ? kModeTensor
                                                               : kModePlain;
}

// Row number k (0 <= k < row_end - row_begin) of a call, counted from
// row_begin up, or with p.reverse from row_end - 1 down.
__device__ __forceinline__ int64_t call_row(const Params& p, int64_t k) {
  return p.reverse ? p.row_end - 1 - k : p.row_begin + k;
}

// ---------------------------------------------------------------------------
// 16-byte packs of eight 2-byte elements
// ---------------------------------------------------------------------------

// kOverflowSq: the square of the smallest magnitude that rounds to infinity
// in the format (bf16: (2 - 2^-8) * 2^127, whose square overflows fp32;
// fp16: 65520).  A row whose fp32 sum of squares stays below it holds no
// element whose rounding to the format overflows.
struct Bf16T {
  static constexpr bool kIsBf16 = true;
  static constexpr float kOverflowSq = 3.40282347e38f;  // FLT_MAX: y^2 overflows first
  static constexpr float kMaxFinite = 3.38953139e38f;   // 0x7f7f
  static __device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);  // round to nearest even
    return *reinterpret_cast<uint32_t*>(&h);
  }
};

struct Fp16T {
  static constexpr bool kIsBf16 = false;
  static constexpr float kOverflowSq = 65520.f * 65520.f;  // exact in fp32
  static constexpr float kMaxFinite = 65504.f;
  static __device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    __half2 h = __floats2half2_rn(lo, hi);  // round to nearest even
    return *reinterpret_cast<uint32_t*>(&h);
  }
};

// acc[i] += element i of the pack, and out[i] = element i + s: each element
// is widened exactly and added with one fp32 rounding, the same result as
// unpack-then-add, in one mixed-precision add (add.rn.f32.bf16 / .f16,
// sm_100) per element.
#define FAR_MIXED_ADD_2(TYPE, ACC0, ACC1, WORD, S0, S1)                                   \
  asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"                           \
      "add.rn.f32." TYPE " %0, lo, %3;\n\tadd.rn.f32." TYPE " %1, hi, %4;\n\t}"           \
      : "=f"(ACC0), "=f"(ACC1)                                                            \
      : "r"(WORD), "f"(S0), "f"(S1))

template <class DT>
__device__ __forceinline__ void add_pack(const uint4& v, float (&acc)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if constexpr (DT::kIsBf16)
      FAR_MIXED_ADD_2("bf16", acc[2 * i], acc[2 * i + 1], w[i], acc[2 * i], acc[2 * i + 1]);
    else
      FAR_MIXED_ADD_2("f16", acc[2 * i], acc[2 * i + 1], w[i], acc[2 * i], acc[2 * i + 1]);
  }
}

template <class DT>
__device__ __forceinline__ void pack_plus(const uint4& v, float s, float (&out)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if constexpr (DT::kIsBf16)
      FAR_MIXED_ADD_2("bf16", out[2 * i], out[2 * i + 1], w[i], s, s);
    else
      FAR_MIXED_ADD_2("f16", out[2 * i], out[2 * i + 1], w[i], s, s);
  }
}

template <class DT>
__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  return make_uint4(DT::pack2(f[0], f[1]), DT::pack2(f[2], f[3]),
                    DT::pack2(f[4], f[5]), DT::pack2(f[6], f[7]));
}

// Four e4m3fn codes (round to nearest even, saturating to +-448), first
// value in the lowest byte.
__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
  const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return lo | (hi << 16);
}

// a / b given inv_b = RN(1/b): q0 = RN(a * inv_b), the exact remainder
// r = a - b*q0 by one FMA, then q0 + r*inv_b rounded once (Markstein's
// FMA-based correction; P. Markstein, "IA-64 and Elementary Functions",
// 2000).  Within one ulp of a/b for normal operands and the correctly
// rounded quotient in all but rare cases, in three instructions and no branch.
__device__ __forceinline__ float div_by(float a, float b, float inv_b) {
  const float q0 = a * inv_b;
  const float r = fmaf(-q0, b, a);
  return fmaf(r, inv_b, q0);
}

// Eight e4m3 codes of o / scale (inv = RN(1/scale); exact: divide exactly,
// for a reciprocal outside the normal range).  A scale of 0 (a per-token row
// of zeros, or one with an inf / NaN input) gives zero codes.
__device__ __forceinline__ uint2 fp8_codes8(const float (&o)[8], float scale, float inv, bool exact) {
  if (scale == 0.f) return make_uint2(0u, 0u);
  float q[8];
  if (exact) {
#pragma unroll
    for (int i = 0; i < 8; ++i) q[i] = __fdiv_rn(o[i], scale);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) q[i] = div_by(o[i], scale, inv);
  }
  return make_uint2(e4m3x4(q[0], q[1], q[2], q[3]), e4m3x4(q[4], q[5], q[6], q[7]));
}

// True when 1 / scale falls outside the normal range, where the quotient is
// taken by an exact division instead.
__device__ __forceinline__ bool needs_exact_div(float scale, float inv) {
  return !(fabsf(inv) < 3.0e38f && fabsf(scale) > 1.0e-37f);
}

// ---------------------------------------------------------------------------
// memory access
// ---------------------------------------------------------------------------

// Partials: read once and never written during the kernel -> non-coherent
// path, no L1 allocation.
__device__ __forceinline__ uint4 ld_once(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
      : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
      : "l"(p));
  return r;
}

// Residual: may be overwritten in place by the same thread afterwards, so
// it takes the coherent path (still without L1 allocation).
__device__ __forceinline__ uint4 ld_once_coherent(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
      : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
      : "l"(p));
  return r;
}

// L2 eviction priorities (PTX createpolicy): per-tensor FP8's first pass
// stores the new residual with evict_last so that as much of it as L2 holds
// is still there when the second pass reads it back, which reads it with
// evict_first (it is not read again).
__device__ __forceinline__ uint64_t l2_evict_last() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ uint64_t l2_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ void st_l2_hint(uint4* p, const uint4& v, uint64_t pol) {
  asm volatile("st.global.L2::cache_hint.v4.u32 [%0], {%1,%2,%3,%4}, %5;"
               ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w), "l"(pol)
               : "memory");
}
// The same through the coherent path, for data written earlier in the same
// kernel.
__device__ __forceinline__ uint4 ld_coherent_l2_hint(const uint4* p, uint64_t pol) {
  uint4 r;
  asm volatile("ld.global.L1::no_allocate.L2::cache_hint.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
      : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
      : "l"(p), "l"(pol));
  return r;
}
__device__ __forceinline__ uint4 ld_once_l2_hint(const uint4* p, uint64_t pol) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
      : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
      : "l"(p), "l"(pol));
  return r;
}

// ---------------------------------------------------------------------------
// TMA bulk copies and mbarriers (PTX ISA: cp.async.bulk, mbarrier)
// ---------------------------------------------------------------------------

// Device-side error word of this library, one per device: bit 0 = a consumer
// gave up waiting for a bulk copy, bit 1 = the producer gave up waiting for
// a free slot, bit 2 = a cluster CTA gave up waiting for its peers' totals,
// bit 3 = a CTA gave up waiting at the per-tensor grid barrier.
// Read and cleared by far_check().
__device__ unsigned int g_far_error = 0u;

constexpr unsigned kErrWaitFull = 1u;
constexpr unsigned kErrWaitEmpty = 2u;
constexpr unsigned kErrWaitPeer = 4u;
constexpr unsigned kErrWaitGrid = 8u;

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return done != 0u;
}

// Wait for the phase of parity `parity` to complete.  Gives up after
// limit_ns, or as soon as *abort is set (when abort is non-null); returns
// false then.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, const volatile int* abort,
                                          uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (abort != nullptr && *abort) return false;
    if (global_ns() - t0 > limit_ns) return false;
  }
}

// As mbar_wait, with cluster-scope acquire (peers arrive on this barrier
// from other CTAs of the cluster); gives up after limit_ns.
__device__ __forceinline__ bool mbar_wait_acquire_cluster(uint64_t* bar, uint32_t parity,
                                                          uint64_t limit_ns) {
  const uint64_t t0 = global_ns();
  for (;;) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    if (done) return true;
    if (global_ns() - t0 > limit_ns) return false;
  }
}

// One 1-D bulk copy global -> this CTA's shared memory, completing `bytes`
// transactions on `bar`.  Both addresses 16-byte aligned, bytes % 16 == 0.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_addr(dst)), "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// The same with an L2 eviction policy for the lines it reads.
__device__ __forceinline__ void bulk_load_hint(void* dst, const void* src, uint32_t bytes,
                                               uint64_t* bar, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;"
      ::"r"(smem_addr(dst)), "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(pol)
      : "memory");
}


// Programmatic dependent launch (PTX griddepcontrol): wait until the grid
// this launch depends on has completed and its writes are visible (a no-op
// without that dependency), then let the next dependent grid be scheduled.
// Called in every kernel before its first access to global memory (only
// shared-memory set-up may come first), so no input is read and no output
// is written before the preceding work in the stream is done.
__device__ __forceinline__ void pdl_enter() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Barrier over the first `nthreads` threads of the CTA (the consumer warps).
__device__ __forceinline__ void consumer_bar(int nthreads) {
  asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
}

// The same barrier, returning whether v held for any of those threads (a
// decision every consumer then takes alike).
__device__ __forceinline__ bool consumer_any(int nthreads, bool v) {
  unsigned r;
  asm volatile(
      "{\n\t.reg .pred q, a;\n\tsetp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred a, 1, %2, q;\n\tselp.u32 %0, 1, 0, a;\n\t}"
      : "=r"(r)
      : "r"(static_cast<unsigned>(v)), "r"(nthreads)
      : "memory");
  return r != 0;
}

// ---------------------------------------------------------------------------
// reductions over one row (all results identical in every thread of the row)
// ---------------------------------------------------------------------------

// Butterfly over `width` lanes: lane i and lane i^m add the same two values,
// so every lane ends with the bit-identical total.
__device__ __forceinline__ float group_sum(float v, int width) {
  for (int m = width >> 1; m > 0; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m, width);
  return v;
}
__device__ __forceinline__ float group_max(float v, int width) {
  for (int m = width >> 1; m > 0; m >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, m, width));
  return v;
}

// A row inside one warp: blockDim.x lanes (a power of two <= 32) per row.
struct SubwarpRed {
  int width;
  __device__ float sum(float v) const { return group_sum(v, width); }
  __device__ float2 sum_max(float s, float m) const {
    return make_float2(group_sum(s, width), group_max(m, width));
  }
  __device__ bool leader() const { return threadIdx.x == 0; }
};

// A row over the whole CTA (blockDim.x a multiple of 32, blockDim.y == 1).
// Each warp reduces, lane 0 parks the warp total in shared memory, and after
// one barrier every warp reduces the same <= 32 totals in the same order.
struct BlockRed {
  float* s_sum;  // [32]
  float* s_max;  // [32]
  __device__ float sum(float v) const {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    v = group_sum(v, 32);
    if (lane == 0) s_sum[warp] = v;
    __syncthreads();
    return group_sum(lane < nw ? s_sum[lane] : 0.f, 32);
  }
  // both totals in one barrier round
  __device__ float2 sum_max(float s, float m) const {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    s = group_sum(s, 32);
    m = group_max(m, 32);
    if (lane == 0) {
      s_sum[warp] = s;
      s_max[warp] = m;
    }
    __syncthreads();
    return make_float2(group_sum(lane < nw ? s_sum[lane] : 0.f, 32),
                       group_max(lane < nw ? s_max[lane] : 0.f, 32));
  }
  __device__ bool leader() const { return threadIdx.x == 0; }
};

// A row over a thread-block cluster.  Each CTA reduces its slice, then
// pushes its totals into slot [rank] of every CTA's shared memory
// (st.shared::cluster) and arrives on that CTA's mbarrier with release
// semantics; each CTA waits (bounded) for all `ncta` arrivals on its own
// mbarrier and reduces the slots in rank order, so every CTA holds the same
// bits.  No CTA touches a peer's shared memory after that peer's arrival
// count is complete, so none can read or write a CTA that has exited.  The
// mbarriers are initialised before the cluster arrive that opens the
// kernel, and the matching cluster wait comes before the first push.
struct ClusterRed {
  BlockRed blk;
  float* s_in;    // [2][16]: pushed sums and maxima, by source rank
  uint64_t* bar;  // counts the ncta pushes
  int ncta;
  int rank;
  uint64_t limit_ns;
  __device__ float2 exchange(float2 t) const {
    asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
    if (threadIdx.x < static_cast<unsigned>(ncta)) {
      const uint32_t dst = static_cast<uint32_t>(threadIdx.x);
      uint32_t rs, rm, rb;
      asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(rs) : "r"(smem_addr(s_in + rank)), "r"(dst));
      asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(rm) : "r"(smem_addr(s_in + 16 + rank)), "r"(dst));
      asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(rb) : "r"(smem_addr(bar)), "r"(dst));
      asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(rs), "f"(t.x) : "memory");
      asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(rm), "f"(t.y) : "memory");
      asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(rb) : "memory");
    }
    if (!mbar_wait_acquire_cluster(bar, 0u, limit_ns)) atomicOr(&g_far_error, kErrWaitPeer);
    const int lane = threadIdx.x & 31;
    const float u = lane < ncta ? s_in[lane] : 0.f;
    const float w = lane < ncta ? s_in[16 + lane] : 0.f;
    return make_float2(group_sum(u, 32), group_max(w, 32));
  }
  __device__ float sum(float v) const { return exchange(make_float2(blk.sum(v), 0.f)).x; }
  __device__ float2 sum_max(float s, float m) const { return exchange(blk.sum_max(s, m)); }
  __device__ bool leader() const { return threadIdx.x == 0 && rank == 0; }
};

// A row over the consumer warps of the ring kernel (a named barrier that
// the producer warp does not join).  `buf` alternates between two halves by
// row parity: a warp can only rewrite a half after every consumer passed the
// next row's barrier, i.e. after everyone finished reading it.
struct RingRed {
  float* buf;     // [2][32]: 0 = sum of squares, 1 = max
  int nthreads;   // consumer threads
  __device__ float sum(float v) const {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = nthreads >> 5;
    v = group_sum(v, 32);
    if (lane == 0) buf[warp] = v;
    consumer_bar(nthreads);
    return group_sum(lane < nw ? buf[lane] : 0.f, 32);
  }
  __device__ float2 sum_max(float s, float m) const {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = nthreads >> 5;
    s = group_sum(s, 32);
    m = group_max(m, 32);
    if (lane == 0) {
      buf[warp] = s;
      buf[32 + warp] = m;
    }
    consumer_bar(nthreads);
    return make_float2(group_sum(lane < nw ? buf[lane] : 0.f, 32),
                       group_max(lane < nw ? buf[32 + lane] : 0.f, 32));
  }
  __device__ bool leader() const { return threadIdx.x == 0; }
};

// ---------------------------------------------------------------------------
// the second half of a row: y (the fp32 sum of partials and residual) is in
// registers; write the new residual, reduce, normalise, quantise.
// This thread owns packs j = j0 + k*jstride (k < VPT) where ok[k].
// ---------------------------------------------------------------------------

// Pack j of gamma: from shared memory where the CTA staged it, else
// through L1 (every row of a CTA reads the same packs).
__device__ __forceinline__ uint4 gamma_pack(const Params& p, const uint4* gamma_smem, int j) {
  return gamma_smem != nullptr ? gamma_smem[j] : __ldg(static_cast<const uint4*>(p.gamma) + j);
}

// MODE (kModePlain / kModeGroup / kModeTensor / kModeTensorNorm): the patterns this
// instantiation serves; per-group and per-tensor code is compiled only into
// their own instantiations, so the other patterns carry none of its registers.
// GPRE: gamma's packs were loaded by the caller into gpre[k] (pack
// j0 + k * jstride); otherwise they come from gamma_smem or through L1.
template <class DT, int VPT, int MODE, bool GPRE, class Red>
__device__ __forceinline__ void finish_row(const Params& p, int64_t row, bool row_ok, int j0,
                                           int jstride, const bool (&ok)[VPT],
                                           float (&y)[VPT][8], const Red& red,
                                           const uint4* gamma_smem, const uint4 (&gpre)[VPT]) {
  const auto gamma_k = [&](int k) -> uint4 {
    if constexpr (GPRE) return gpre[k];
    else return gamma_pack(p, gamma_smem, j0 + k * jstride);
  };
  const int64_t rbase = row * static_cast<int64_t>(p.packs);  // first pack of the row
  // dynamic per-tensor FP8 runs in two passes: the first records rinv and
  // the call's amax (and the new residual or norm_out the second pass reads);
  // the second writes the other outputs
  const bool tensor_amax = is_tensor_mode(MODE) && p.pattern == kTensorAmax;
  const bool tensor_quant = is_tensor_mode(MODE) && p.pattern == kTensorQuant;
  if (p.residual_out != nullptr && !tensor_amax) {
#pragma unroll
    for (int k = 0; k < VPT; ++k)
      if (ok[k]) static_cast<uint4*>(p.residual_out)[rbase + j0 + k * jstride] = pack8<DT>(y[k]);
  }

  // a3: mean of squares; pairwise inside the thread, butterflies above it.
  float sq[VPT];
#pragma unroll
  for (int k = 0; k < VPT; ++k) {
    const float a = y[k][0] * y[k][0] + y[k][1] * y[k][1];
    const float b = y[k][2] * y[k][2] + y[k][3] * y[k][3];
    const float c = y[k][4] * y[k][4] + y[k][5] * y[k][5];
    const float d = y[k][6] * y[k][6] + y[k][7] * y[k][7];
    sq[k] = (a + b) + (c + d);
  }
#pragma unroll
  for (int w = 1; w < VPT; w <<= 1)
#pragma unroll
    for (int k = 0; k + w < VPT; k += 2 * w) sq[k] += sq[k + w];

  const bool fp8_static = p.pattern == kFp8Static;
  const bool fp8_token = p.pattern == kFp8Token;
  constexpr bool fp8_group = MODE == kModeGroup;

  // a5b needs max|o| = rinv * max|y * (gamma + wb)| (rinv > 0): its local
  // part goes into the same reduction round as the sum of squares.  The
  // second per-tensor pass reuses the first pass's rinv: no reduction.
  // Per-token keeps y * (gamma + wb) in y (one read of gamma per row), so
  // its o is (y * g) * rinv; the other patterns form (y * rinv) * g below.
  float ss = 0.f, gmax = 0.f;
  if (fp8_token || tensor_amax) {
    float m = 0.f;
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
      if (!ok[k]) continue;
      float g[8];
      pack_plus<DT>(gamma_k(k), p.weight_bias, g);
      if (fp8_token) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          y[k][i] *= g[i];
          m = fmaxf(m, fabsf(y[k][i]));
        }
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(y[k][i] * g[i]));
      }
    }
    const float2 r = red.sum_max(sq[0], m);
    ss = r.x;
    gmax = r.y;
  } else if (!tensor_quant) {
    ss = red.sum(sq[0]);
  }
  // (a row past the end of the call, in a CTA of several rows, reads nothing;
  // the stored rinv carries the first pass's row flag in its sign bit)
  const float rinv = tensor_quant ? (row_ok ? fabsf(p.ws_rinv[row - p.ws_row0]) : 0.f)
                                  : __frsqrt_rn(__fdiv_rn(ss, static_cast<float>(p.H)) + p.eps);

  if (tensor_amax) {
    // A row whose sum of squares reaches the square of the format's overflow
    // threshold (or is inf / NaN) may hold an element that rounds to
    // infinity: the second pass must rebuild its y from the inputs, so its
    // new residual is not stored here and the row is flagged (sign bit of
    // the stored rinv, which is otherwise +0, positive or +inf).
    // With norm_out stored for the second pass, a row whose amax reaches
    // the format's largest finite value (an element of norm_out may be
    // infinite) is flagged too.  norm_out is written here for every row;
    // the new residual of a flagged row is left to the second pass (which
    // rebuilds the row from the inputs, the residual possibly among them).
    bool rebuild = !(ss < DT::kOverflowSq);
    if (MODE == kModeTensor && p.tensor_source == 1 && !rebuild) {
      const uint64_t keep = l2_evict_last();
#pragma unroll
      for (int k = 0; k < VPT; ++k)
        if (ok[k]) st_l2_hint(static_cast<uint4*>(p.residual_out) + rbase + j0 + k * jstride, pack8<DT>(y[k]), keep);
    }
    if constexpr (MODE == kModeTensorNorm) {
      rebuild = rebuild || !(rinv * gmax < DT::kMaxFinite);
      const uint64_t keep = l2_evict_last();
#pragma unroll
      for (int k = 0; k < VPT; ++k) {
        if (!ok[k]) continue;
        const int64_t pk = rbase + j0 + k * jstride;
        if (p.residual_out != nullptr && !rebuild) static_cast<uint4*>(p.residual_out)[pk] = pack8<DT>(y[k]);
        float g[8];
        pack_plus<DT>(gamma_k(k), p.weight_bias, g);
        float o[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i] = (y[k][i] * rinv) * g[i];
        st_l2_hint(static_cast<uint4*>(p.norm_out) + pk, pack8<DT>(o), keep);
      }
    }
    if (row_ok && red.leader()) {
      p.ws_rinv[row - p.ws_row0] =
          __uint_as_float(__float_as_uint(rinv) | (rebuild ? 0x80000000u : 0u));
      // non-negative floats order like their bit patterns; a row whose rinv
      // is 0 or NaN (inf / NaN input) has no finite nonzero o: it adds nothing
      const float a = rinv * gmax;
      if (a == a) atomicMax(p.ws_amax, __float_as_uint(a));
    }
    return;
  }

  // the divisor of the FP8 codes: the static scale, or max|o| / 448 of the
  // row or of the call
  float scale = 1.f;
  if (fp8_static) scale = __ldg(p.scale_in);
  if (fp8_token || tensor_quant) {
    scale = __fdiv_rn(fp8_token ? rinv * gmax : __uint_as_float(*p.ws_amax), 448.f);
    // a row with an inf or NaN input has rinv 0 or NaN; its finite o are 0
    // and the rest NaN, which take no part in the amax: scale 0
    if (scale != scale) scale = 0.f;
    if (row_ok && red.leader() && (fp8_token || row == p.ws_row0))
      p.scale_out[fp8_token ? row : 0] = scale;
  }
  const float inv = __frcp_rn(scale);
  // outside the reciprocal's normal range, divide exactly (uniform per row)
  const bool exact = needs_exact_div(scale, inv);

  // a4: o = y * rinv * (gamma + weight_bias); a5: FP8 codes.
#pragma unroll
  for (int k = 0; k < VPT; ++k) {
    if (!ok[k]) continue;
    const int64_t pk = rbase + j0 + k * jstride;
    if (fp8_token) {  // y already holds y * (gamma + wb)
#pragma unroll
      for (int i = 0; i < 8; ++i) y[k][i] *= rinv;
    } else {
      float g[8];  // gamma + weight_bias in fp32
      pack_plus<DT>(gamma_k(k), p.weight_bias, g);
#pragma unroll
      for (int i = 0; i < 8; ++i) y[k][i] = (y[k][i] * rinv) * g[i];
    }
    if (p.norm_out != nullptr) static_cast<uint4*>(p.norm_out)[pk] = pack8<DT>(y[k]);
    if (fp8_static || fp8_token || tensor_quant)  // (per-group codes: below)
      reinterpret_cast<uint2*>(p.quant_out)[pk] = fp8_codes8(y[k], scale, inv, exact);
  }

  // a5d: per-group FP8.  A group is p.group_lanes consecutive packs of the
  // row, held by as many consecutive lanes of one warp (the pack index is
  // lane-contiguous and warp-aligned in every kernel that takes this
  // pattern), so its amax is a shuffle butterfly over those lanes; every
  // lane takes part before any lane skips its store.
  if constexpr (fp8_group) {
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
      float m = 0.f;
      if (ok[k]) {
#pragma unroll
        for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(y[k][i]));
      }
      m = group_max(m, p.group_lanes);
      if (!ok[k]) continue;
      const int jpk = j0 + k * jstride;  // pack index in the row
      const float sc = __fdiv_rn(m, 448.f);
      // group_lanes is a power of two: its group is jpk >> log2(group_lanes)
      if (row_ok && (jpk & (p.group_lanes - 1)) == 0)
        p.scale_out[row * p.groups_per_row + (jpk >> (__ffs(p.group_lanes) - 1))] = sc;
      const float inv_g = __frcp_rn(sc);
      reinterpret_cast<uint2*>(p.quant_out)[rbase + jpk] =
          fp8_codes8(y[k], sc, inv_g, needs_exact_div(sc, inv_g));
    }
  }
}

// ---------------------------------------------------------------------------
// one row (or one slice of it) straight from global memory into registers:
// packs j = j0 + k*jstride, k < VPT, j < jend
// ---------------------------------------------------------------------------

// Loads are issued ahead of their use so that a short call waits on about
// one memory round trip per row, not one per batch of partials plus one for
// the residual and one for gamma: the residual and gamma (read after the
// reduction) go out with the first batch of partials, and at up to 4 packs
// per thread each batch is folded in only after the next batch's loads are
// issued.  kBatch partials per batch keep the loads in flight within the
// kernels' register budgets.
template <int VPT>
struct RowLoads {
  static constexpr int kBatch = VPT <= 2 ? 4 : (VPT == 4 ? 1 : 4);
  static constexpr bool kPipelined = VPT <= 4;
  static constexpr bool kGammaAhead = VPT <= 4;
};

template <class DT, int VPT, int MODE, class Red>
__device__ __forceinline__ void fused_row(const Params& p, int64_t row, bool row_ok,
                                          int j0, int jstride, int jend, const Red& red) {
  using L = RowLoads<VPT>;
  constexpr int B = L::kBatch;
  const int64_t rbase = row * static_cast<int64_t>(p.packs);  // first pack of the row
  float y[VPT][8];
  bool ok[VPT];
#pragma unroll
  for (int k = 0; k < VPT; ++k) {
    ok[k] = row_ok && (j0 + k * jstride) < jend;
#pragma unroll
    for (int i = 0; i < 8; ++i) y[k][i] = 0.f;
  }
  const auto load_batch = [&](uint4 (&v)[B][VPT], int r0) {
#pragma unroll
    for (int c = 0; c < B; ++c) {
#pragma unroll
      for (int k = 0; k < VPT; ++k) {
        v[c][k] = make_uint4(0u, 0u, 0u, 0u);
        if (r0 + c < p.W && ok[k])
          v[c][k] = ld_once(static_cast<const uint4*>(p.partials[r0 + c]) + rbase + j0 + k * jstride);
      }
    }
  };

  // a1 (first batch), a2's residual and gamma, all in flight together
  uint4 cur[B][VPT], res[VPT], gam[VPT];
  load_batch(cur, 0);
#pragma unroll
  for (int k = 0; k < VPT; ++k) {
    res[k] = make_uint4(0u, 0u, 0u, 0u);
    if (p.residual != nullptr && ok[k])
      res[k] = ld_once_coherent(static_cast<const uint4*>(p.residual) + rbase + j0 + k * jstride);
    if constexpr (L::kGammaAhead)
      gam[k] = ok[k] ? __ldg(static_cast<const uint4*>(p.gamma) + j0 + k * jstride)
                     : make_uint4(0u, 0u, 0u, 0u);
  }

  // a1: sum the W partials in fp32 in order 0..W-1
  for (int r0 = 0; r0 < p.W; r0 += B) {
    if constexpr (L::kPipelined) {
      uint4 nxt[B][VPT];
      const bool more = r0 + B < p.W;
      if (more) load_batch(nxt, r0 + B);
#pragma unroll
      for (int c = 0; c < B; ++c) {
#pragma unroll
        for (int k = 0; k < VPT; ++k) add_pack<DT>(cur[c][k], y[k]);
      }
      if (more) {
#pragma unroll
        for (int c = 0; c < B; ++c) {
#pragma unroll
          for (int k = 0; k < VPT; ++k) cur[c][k] = nxt[c][k];
        }
      }
    } else {
      if (r0 > 0) load_batch(cur, r0);
#pragma unroll
      for (int c = 0; c < B; ++c) {
#pragma unroll
        for (int k = 0; k < VPT; ++k) add_pack<DT>(cur[c][k], y[k]);
      }
    }
  }

  // a2: add the residual (a zero pack without one: y + 0 = y, y is never -0)
  if (p.residual != nullptr) {
#pragma unroll
    for (int k = 0; k < VPT; ++k) add_pack<DT>(res[k], y[k]);
  }
  finish_row<DT, VPT, MODE, L::kGammaAhead>(p, row, row_ok, j0, jstride, ok, y, red, nullptr, gam);
}

// ---------------------------------------------------------------------------
// kernels
// ---------------------------------------------------------------------------

// Prefill: blockDim = (tpr, rows_per_cta).  SUB: a row lives inside one warp
// (tpr <= 32, power of two); otherwise one row per CTA.
// Registers: at one pack per thread (rows of at most 256 packs, often short
// calls of many rows) four 256-thread CTAs per SM; otherwise two, one at 8.
template <class DT, int VPT, bool SUB, int MODE>
__global__ void __launch_bounds__(kMaxThreads, (VPT >= 8 ? 1 : (VPT == 1 ? 4 : 2)))
far_prefill_kernel(const Params p) {
  pdl_enter();
  const int64_t k = static_cast<int64_t>(blockIdx.x) * blockDim.y + threadIdx.y;
  const bool row_ok = k < p.row_end - p.row_begin;
  const int64_t row = call_row(p, k);
  if constexpr (SUB) {
    const SubwarpRed red{static_cast<int>(blockDim.x)};
    fused_row<DT, VPT, MODE>(p, row, row_ok, threadIdx.x, blockDim.x, p.packs, red);
  } else {
    __shared__ float s_sum[32], s_max[32];
    const BlockRed red{s_sum, s_max};
    fused_row<DT, VPT, MODE>(p, row, row_ok, threadIdx.x, blockDim.x, p.packs, red);
  }
}

// Decode: grid = (cluster, rows), one cluster per row; CTA `rank` of the
// cluster takes packs [rank*chunk, min(packs, (rank+1)*chunk)).
template <class DT, int VPT>
__global__ void __launch_bounds__(kMaxThreads, (VPT >= 8 ? 1 : 2))
far_decode_kernel(const Params p) {
  // the shared-memory set-up touches no global memory: it runs before the
  // wait for the preceding grid, overlapping its tail
  __shared__ float s_sum[32], s_max[32], s_in[32];
  __shared__ uint64_t s_bar;
  cg::cluster_group cl = cg::this_cluster();
  const int rank = static_cast<int>(cl.block_rank());
  const int ncta = static_cast<int>(cl.num_blocks());
  if (threadIdx.x == 0) {
    mbar_init(&s_bar, static_cast<uint32_t>(ncta));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
  pdl_enter();
  const int64_t row = call_row(p, blockIdx.y);
  const int chunk = (p.packs + ncta - 1) / ncta;
  const int jbeg = rank * chunk;
  const int jend = min(p.packs, jbeg + chunk);
  const ClusterRed red{BlockRed{s_sum, s_max}, s_in, &s_bar, ncta, rank, p.wait_limit_ns};
  const bool row_ok = blockIdx.y < p.row_end - p.row_begin;
  fused_row<DT, VPT, kModePlain>(p, row, row_ok, jbeg + static_cast<int>(threadIdx.x), blockDim.x, jend,
                            red);
}

// ---------------------------------------------------------------------------
// dynamic per-tensor FP8: the codes from the stored new residual
// ---------------------------------------------------------------------------

// The 8 codes of one pack.  In the usual case (a scale whose reciprocal is
// normal) the quotient is formed as q = (y * (rinv / scale)) * (gamma + wb),
// two multiplies per element with rs = RN(rinv * RN(1 / scale)) per row: a
// few fp32 ulps from o / scale, nothing against the half-ulp of the 2-byte
// format already in y here and far inside one e4m3 step.  Otherwise o is
// formed and divided as in every other pattern.
template <class DT>
__device__ __forceinline__ uint2 tensor_codes(const uint4& gam, float wb, float (&y)[8], float rinv,
                                              float rs, float scale, float inv, bool exact) {
  float g[8];
  pack_plus<DT>(gam, wb, g);
  if (!exact && scale != 0.f) {
#pragma unroll
    for (int i = 0; i < 8; ++i) y[i] = (y[i] * rs) * g[i];
    return make_uint2(e4m3x4(y[0], y[1], y[2], y[3]), e4m3x4(y[4], y[5], y[6], y[7]));
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) y[i] = (y[i] * rinv) * g[i];
  return fp8_codes8(y, scale, inv, exact);
}

// A pack of eight 1.0 in the 2-byte format: with weight_bias 0 and rinv 1,
// tensor_codes then forms the codes of the pack it is given as o itself
// (norm_out read back: o within half an ulp of the 2-byte format), by the
// same instructions as the codes of round(y).
template <class DT>
__device__ __forceinline__ uint4 ones_pack() {
  const uint32_t one2 = DT::kIsBf16 ? 0x3F803F80u : 0x3C003C00u;
  return make_uint4(one2, one2, one2, one2);
}

// The 8 codes of one pack from what the first pass stored: the new residual
// round(y) (tensor_source 1: o formed as above) or norm_out round(o)
// (tensor_source 2: o itself).
template <class DT>
__device__ __forceinline__ uint2 stored_codes(int source, const uint4& v, const uint4& gam, float wb,
                                              float rinv, float rs, float scale, float inv,
                                              bool exact) {
  float x[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  add_pack<DT>(v, x);  // 0 + x: the 2-byte value widened exactly
  const bool o = source == 2;
  return tensor_codes<DT>(o ? ones_pack<DT>() : gam, o ? 0.f : wb, x, o ? 1.f : rinv, o ? inv : rs,
                          scale, inv, exact);
}

// One row of the second pass on its own: from the stored new residual, or
// (a flagged row) rebuilt from the inputs in the first pass's order --
// partials 0..W-1, then the residual -- with its new residual written here.
// COHERENT: the stored new residual was written earlier in the same kernel
// (the fused form), so it is read through the coherent path; gamma_s: gamma
// staged in shared memory, or null (read through L1).
template <class DT, int VPT, bool COHERENT = false>
__device__ __forceinline__ void tensor_quant_row(const Params& p, int64_t row, float w, int j0,
                                                 int tpr, const bool (&ok)[VPT], float inv,
                                                 float scale, bool exact, uint64_t drop,
                                                 const uint4* gamma_s = nullptr) {
  const uint4* gamma = gamma_s != nullptr ? gamma_s : static_cast<const uint4*>(p.gamma);
  const int64_t rbase = row * static_cast<int64_t>(p.packs);
  const bool rebuild = signbit(w);
  const float rinv = fabsf(w);
  const float rs = rinv * inv;
#pragma unroll
  for (int q = 0; q < VPT; ++q) {
    if (!ok[q]) continue;
    const int64_t pk = rbase + j0 + q * tpr;
    const uint4 g = gamma_s != nullptr ? gamma[j0 + q * tpr] : __ldg(gamma + j0 + q * tpr);
    if (!rebuild) {
      const uint4* src = static_cast<const uint4*>(p.tensor_source == 2 ? p.norm_out : p.residual_out) + pk;
      reinterpret_cast<uint2*>(p.quant_out)[pk] = stored_codes<DT>(
          p.tensor_source, COHERENT ? ld_coherent_l2_hint(src, drop) : ld_once_l2_hint(src, drop), g,
          p.weight_bias, rinv, rs, scale, inv, exact);
      continue;
    }
    float y[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int r = 0; r < p.W; ++r) add_pack<DT>(ld_once(static_cast<const uint4*>(p.partials[r]) + pk), y);
    if (p.residual != nullptr)
      add_pack<DT>(ld_once_coherent(static_cast<const uint4*>(p.residual) + pk), y);
    if (p.residual_out != nullptr) static_cast<uint4*>(p.residual_out)[pk] = pack8<DT>(y);
    reinterpret_cast<uint2*>(p.quant_out)[pk] =
        tensor_codes<DT>(g, p.weight_bias, y, rinv, rs, scale, inv, exact);
  }
}

// The scale of dynamic per-tensor FP8 from the call's amax word, and the
// derived divisor terms (see tensor_codes).  CTA 0 writes scale_out[0].
struct TensorScale {
  float scale, inv;
  bool exact;
  __device__ explicit TensorScale(const Params& p, unsigned amax_bits) {
    scale = __fdiv_rn(__uint_as_float(amax_bits), 448.f);
    if (scale != scale) scale = 0.f;
    if (blockIdx.x == 0 && threadIdx.x == 0 && threadIdx.y == 0) p.scale_out[0] = scale;
    inv = __frcp_rn(scale);
    exact = needs_exact_div(scale, inv);
  }
};

// The fused per-tensor form's grid barrier, run by the consumer threads of a
// ring CTA once it has taken no more rows: the CTA adds the rows it did to
// the call's count, then waits until every row of the call is done, when
// the call's amax is final.  It waits for rows, not for CTAs: a CTA that
// has not started holds no row, so the wait needs no co-residency of the
// grid.  The wait is bounded; a CTA that gives up sets the device error
// word and its abort flag (it writes no codes).  Returns false then.
__device__ __forceinline__ bool tensor_grid_barrier(const Params& p, int ncons,
                                                    volatile int* abort_flag, int64_t rows_done) {
  consumer_bar(ncons);  // every consumer of this CTA is past its last row
  if (threadIdx.x == 0) {
    __threadfence();    // this CTA's amax and rows before its count (cumulative)
    atomicAdd(p.ws_done, static_cast<unsigned>(rows_done));
    const unsigned nrows = static_cast<unsigned>(p.row_end - p.row_begin);
    const uint64_t t0 = global_ns();
    for (;;) {
      unsigned n;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(n) : "l"(p.ws_done) : "memory");
      if (n >= nrows) break;
      if (global_ns() - t0 > p.wait_limit_ns) {
        atomicOr(&g_far_error, kErrWaitGrid);
        *abort_flag = 1;
        break;
      }
    }
  }
  consumer_bar(ncons);
  return !*abort_flag;
}

// Barrier between the consumers and the whole producer warp of a ring CTA.
__device__ __forceinline__ void tail_bar(int nthreads) {
  asm volatile("bar.sync 2, %0;" ::"r"(nthreads) : "memory");
}

// Prefill through the TMA engine: a persistent CTA per SM (or two) walks
// rows blockIdx.x, blockIdx.x + gridDim.x, ...  Its last warp is the producer:
// one thread streams each row's W partial segments and its residual segment
// (H*2 bytes each) with cp.async.bulk into a ring of `nslot` shared-memory
// slots, running up to nslot segments ahead.  The first `ncons` threads are
// consumers: they wait for a slot (mbarrier, transaction count), fold its
// packs into their fp32 row registers in the same order as the direct path
// (partials 0..W-1, then the residual), release the slot, and finish the row
// from registers.  The bytes in flight live in shared memory, not in
// registers, so each SM keeps ~100-200 KB of loads outstanding.
//
// Every wait is bounded (p.wait_limit_ns, 2 s); a wait that gives up sets the
// device error word and the CTA's abort flag, after which no wait blocks,
// the producer stops, and thread 0 waits (bounded) for the copies already
// issued before the CTA exits.
// MINB: CTAs per SM the register budget is sized for (2 or 3; 1 or 2 at VPT 8).
// MAXC: most consumer threads (the wide build: kRingWideConsumers).
template <class DT, int VPT, int MINB, int MODE, int MAXC = kRingMaxConsumers>
__global__ void __launch_bounds__(MAXC + 32, MINB)
far_ring_kernel(const Params p, int nslot, int ncons, int stage_gamma) {
  extern __shared__ __align__(128) unsigned char smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + nslot;
  RingHeader* hdr = reinterpret_cast<RingHeader*>(empty + nslot);
  volatile int* abort_flag = &hdr->abort;
  volatile int* producer_done = &hdr->producer_done;
  volatile long long* issued_count = &hdr->issued;
  const uint32_t seg_bytes = static_cast<uint32_t>(p.H) * 2u;
  // gamma, when staged, sits between the header and the slots
  uint4* gamma_s = stage_gamma ? reinterpret_cast<uint4*>(smem + ring_offset(nslot)) : nullptr;
  unsigned char* ring = smem + ring_offset(nslot) + (stage_gamma ? seg_bytes : 0u);
  const int S = p.W + (p.residual != nullptr ? 1 : 0);
  const int64_t nrows = p.row_end - p.row_begin;
  const int64_t my_rows = (nrows - blockIdx.x + gridDim.x - 1) / gridDim.x;

  if (threadIdx.x == 0) {
    for (int i = 0; i < nslot; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], static_cast<uint32_t>(ncons / 32));
    }
    *abort_flag = 0;
    *producer_done = 0;
    *issued_count = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();  // the mbarriers are ready: the producer may start at once
  // everything above touches shared memory only: it runs before the wait for
  // the preceding grid, overlapping its tail
  pdl_enter();

  if (threadIdx.x >= ncons) {
    // producer warp: one thread issues, the rest of the warp is idle.
    // Copy g goes to slot g mod nslot, whose use count parity is `phase`
    // (counters, not 64-bit divisions).
    int slot = 0;
    uint32_t phase = 0;
    int64_t issued = 0;
    if (threadIdx.x == ncons) {
      // per-tensor FP8 reading back its new residual: the inputs, read
      // once, leave L2 first, so that the new residual (stored evict-last)
      // is what L2 keeps for the second pass
      const bool drop_inputs = is_tensor_mode(MODE) && p.tensor_source != 0;
      uint64_t drop = 0;
      if constexpr (is_tensor_mode(MODE)) drop = l2_evict_first();
      // Rows: ordinals blockIdx.x + i * gridDim.x; or, in the fused
      // per-tensor form, taken one at a time from the call's counter (the
      // next one claimed while this one's segments are issued), so that the
      // CTAs reach the grid barrier together.  Then the slot of a row's
      // first segment names the row, and a slot naming -1, completed
      // without a copy, ends the consumers' first pass.
      bool dyn = false;
      if constexpr (is_tensor_mode(MODE)) dyn = p.tensor_fused != 0;
      int64_t ord = dyn ? static_cast<int64_t>(atomicAdd(p.ws_claim, 1u)) : blockIdx.x;
      int64_t g = 0;  // copies issued
      for (int64_t i = 0; !*abort_flag; ++i) {
        const bool more = dyn ? ord < nrows : i < my_rows;
        if (!more && !dyn) break;
        int64_t next = 0;
        if (dyn && more) next = atomicAdd(p.ws_claim, 1u);
        const int nk = more ? S : 1;  // the end marker takes one slot
        bool stop = false;
        for (int k = 0; k < nk; ++k) {
          if (!mbar_wait(&empty[slot], phase ^ 1u, abort_flag, p.wait_limit_ns)) {
            if (!*abort_flag) atomicOr(&g_far_error, kErrWaitEmpty);
            *abort_flag = 1;
            stop = true;
            break;
          }
          if (dyn && k == 0) hdr->slot_row[slot] = more ? static_cast<int>(ord) : -1;
          if (!more) {
            mbar_arrive(&full[slot]);
          } else {
            if (g != p.stall_segment) {  // test hook: that copy is never issued
              const void* base = (k < p.W) ? p.partials[k] : p.residual;
              const unsigned char* src = static_cast<const unsigned char*>(base) +
                                         call_row(p, ord) * static_cast<int64_t>(seg_bytes);
              mbar_arrive_expect_tx(&full[slot], seg_bytes);
              if (drop_inputs)
                bulk_load_hint(ring + static_cast<size_t>(slot) * seg_bytes, src, seg_bytes, &full[slot], drop);
              else
                bulk_load(ring + static_cast<size_t>(slot) * seg_bytes, src, seg_bytes, &full[slot]);
            }
            ++g;
          }
          ++issued;
          if (++slot == nslot) {
            slot = 0;
            phase ^= 1u;
          }
        }
        if (stop || !more) break;
        ord = dyn ? next : ord + gridDim.x;
      }
    }
    if constexpr (is_tensor_mode(MODE)) {
      // The fused per-tensor form: once every CTA has stored its rows' new
      // residuals and flags (fenced for the async proxy) and the consumers
      // are past the grid barrier, stream the rows back through the ring:
      // the stored row, or for a flagged row all its input segments.  Rows
      // are taken in chunks of p.tail_chunk ordinals, the highest ordinals
      // (taken last in the first pass, so the likeliest in L2) first: about
      // three quarters in fixed rounds, the rest from a second counter, so
      // that a CTA whose SM drains its ring faster takes more of the last
      // rows.
      // The slot of a row's first segment names the row and holds its stored
      // rinv (sign bit: the flag); a slot naming -1, completed without a
      // copy, ends the second pass.  The next chunk is claimed while this
      // one is issued, and its flags are read (one row per lane) once this
      // one is issued, while the ring still holds nslot segments.
      if (p.tensor_fused) {
        tail_bar(ncons + 32);
        const int lane = threadIdx.x - ncons;
        const uint64_t drop_tail = l2_evict_first();
        const int64_t C = p.tail_chunk;
        // about three quarters of the rows are dealt out in fixed rounds
        // (CTA b takes chunk b of each round): no claim round trip for
        // them; the counter deals out the rest, which evens out the ends
        const int64_t G = gridDim.x;
        int64_t rounds = (3 * nrows / 4) / (G * C);
        if (rounds < 1) rounds = 1;
        const int64_t first_dealt = rounds * G * C;
        int64_t dealt = 0;  // fixed rounds taken so far
        const auto claim = [&]() -> int64_t {
          if (dealt < rounds) return (dealt++ * G + blockIdx.x) * C;
          unsigned b = 0;
          if (lane == 0) b = atomicAdd(p.ws_claim2, static_cast<unsigned>(C));
          return first_dealt + static_cast<int64_t>(__shfl_sync(0xffffffffu, b, 0));
        };
        const auto flags = [&](int64_t b) -> float {
          float w = 0.f;
          if (lane < C && b + lane < nrows) {
            const int64_t r = call_row(p, nrows - 1 - (b + lane));
            w = *reinterpret_cast<volatile const float*>(p.ws_rinv + (r - p.ws_row0));
          }
          return w;
        };
        int64_t base = claim();
        float w = flags(base);
        int64_t next = claim();
        bool stop = false;
        while (!stop) {
          if (__shfl_sync(0xffffffffu, lane == 0 ? *abort_flag : 0, 0)) break;
          if (base >= nrows) {
            // the end marker
            if (lane == 0) {
              if (mbar_wait(&empty[slot], phase ^ 1u, abort_flag, p.wait_limit_ns)) {
                hdr->slot_row[slot] = -1;
                mbar_arrive(&full[slot]);
                ++issued;
                if (++slot == nslot) {
                  slot = 0;
                  phase ^= 1u;
                }
              } else {
                if (!*abort_flag) atomicOr(&g_far_error, kErrWaitEmpty);
                *abort_flag = 1;
              }
            }
            break;
          }
          for (int j = 0; j < C; ++j) {
            const float wj = __shfl_sync(0xffffffffu, w, j);
            if (lane == 0 && !stop && base + j < nrows) {
              const int64_t ord = nrows - 1 - (base + j);
              const int64_t row = call_row(p, ord);
              const bool rebuild = signbit(wj);
              const int nseg = rebuild ? S : 1;
              for (int k = 0; k < nseg; ++k) {
                if (!mbar_wait(&empty[slot], phase ^ 1u, abort_flag, p.wait_limit_ns)) {
                  if (!*abort_flag) atomicOr(&g_far_error, kErrWaitEmpty);
                  *abort_flag = 1;
                  stop = true;
                  break;
                }
                if (k == 0) {
                  hdr->slot_row[slot] = static_cast<int>(ord);
                  hdr->slot_w[slot] = wj;
                }
                const void* stored = MODE == kModeTensorNorm ? p.norm_out : p.residual_out;
                const void* src = !rebuild ? stored : (k < p.W ? p.partials[k] : p.residual);
                mbar_arrive_expect_tx(&full[slot], seg_bytes);
                bulk_load_hint(ring + static_cast<size_t>(slot) * seg_bytes,
                               static_cast<const unsigned char*>(src) + row * static_cast<int64_t>(seg_bytes),
                               seg_bytes, &full[slot], drop_tail);
                ++issued;
                if (++slot == nslot) {
                  slot = 0;
                  phase ^= 1u;
                }
              }
            }
          }
          stop = __shfl_sync(0xffffffffu, stop ? 1 : 0, 0) != 0;
          base = next;
          w = flags(base);
          next = claim();
        }
      }
    }
    if (threadIdx.x == ncons) {
      *issued_count = issued;  // read by the drain below
      __threadfence_block();
      *producer_done = 1;
    }
    return;
  }

  // consumers.  gamma is read once per CTA into shared memory while the
  // producer issues its first copies; the consumers' barrier orders the
  // staging before the first row's use of it.
  if (stage_gamma) {
    for (int j = threadIdx.x; j < p.packs; j += ncons)
      gamma_s[j] = __ldg(static_cast<const uint4*>(p.gamma) + j);
    consumer_bar(ncons);
  }
  const RingRed red0{&hdr->red[0][0][0], ncons}, red1{&hdr->red[1][0][0], ncons};
  const uint4 no_gamma[VPT] = {};  // gamma comes from shared memory or L1 here
  const int j0 = threadIdx.x;
  int slot = 0;  // the slot of the next segment and its use count parity
  uint32_t phase = 0;
  bool dyn = false;  // rows named by the producer (the fused per-tensor form)
  if constexpr (is_tensor_mode(MODE)) dyn = p.tensor_fused != 0;
  int64_t i = 0;  // rows done
  for (;; ++i) {
    int64_t ord;
    if (dyn) {
      // the row is named in the slot of its first segment; every consumer
      // leaves the loop alike, at the end marker or after a wait gave up
      if (!*abort_flag && !mbar_wait(&full[slot], phase, abort_flag, p.wait_limit_ns)) {
        if (!*abort_flag) atomicOr(&g_far_error, kErrWaitFull);
        *abort_flag = 1;
      }
      const int named = hdr->slot_row[slot];
      if (consumer_any(ncons, named < 0 || *abort_flag)) {
        __syncwarp();
        if ((threadIdx.x & 31) == 0) mbar_arrive(&empty[slot]);
        if (++slot == nslot) {
          slot = 0;
          phase ^= 1u;
        }
        break;
      }
      ord = named;
    } else {
      if (i >= my_rows) break;
      ord = blockIdx.x + i * gridDim.x;
    }
    const int64_t row = call_row(p, ord);
    float y[VPT][8];
    bool ok[VPT];
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
      ok[k] = (j0 + k * ncons) < p.packs;
#pragma unroll
      for (int e = 0; e < 8; ++e) y[k][e] = 0.f;
    }
    for (int k = 0; k < S; ++k) {
      if (!(dyn && k == 0) && !*abort_flag &&
          !mbar_wait(&full[slot], phase, abort_flag, p.wait_limit_ns)) {
        if (!*abort_flag) atomicOr(&g_far_error, kErrWaitFull);
        *abort_flag = 1;
      }
      const uint4* seg = reinterpret_cast<const uint4*>(ring + static_cast<size_t>(slot) * seg_bytes);
#pragma unroll
      for (int q = 0; q < VPT; ++q)
        if (ok[q]) add_pack<DT>(seg[j0 + q * ncons], y[q]);
      __syncwarp();
      if ((threadIdx.x & 31) == 0) mbar_arrive(&empty[slot]);
      if (++slot == nslot) {
        slot = 0;
        phase ^= 1u;
      }
    }
    finish_row<DT, VPT, MODE, false>(p, row, true, j0, ncons, ok, y, (i & 1) ? red1 : red0,
                                      gamma_s, no_gamma);
  }
  if constexpr (is_tensor_mode(MODE)) {
    if (p.tensor_fused) {
      // this thread's new-residual stores, before any CTA's bulk copies read them
      asm volatile("fence.proxy.async.global;" ::: "memory");
      const bool passed = tensor_grid_barrier(p, ncons, abort_flag, i);
      tail_bar(ncons + 32);  // the producer starts the second pass
      if (passed) {
        unsigned amax_bits;
        asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(amax_bits) : "l"(p.ws_amax) : "memory");
        const TensorScale ts(p, amax_bits);
        // rows as the producer names them, each with its stored rinv, until
        // the end marker (or a wait that gave up: every warp leaves alike)
        for (;;) {
          if (!*abort_flag && !mbar_wait(&full[slot], phase, abort_flag, p.wait_limit_ns)) {
            if (!*abort_flag) atomicOr(&g_far_error, kErrWaitFull);
            *abort_flag = 1;
          }
          const int named = hdr->slot_row[slot];
          const float w = hdr->slot_w[slot];
          if (__any_sync(0xffffffffu, named < 0 || *abort_flag)) {
            __syncwarp();
            if ((threadIdx.x & 31) == 0) mbar_arrive(&empty[slot]);
            if (++slot == nslot) {
              slot = 0;
              phase ^= 1u;
            }
            break;
          }
          const int64_t row = call_row(p, named);
          const bool rebuild = signbit(w);
          const int nseg = rebuild ? S : 1;
          float y[VPT][8];
          bool ok[VPT];
#pragma unroll
          for (int q = 0; q < VPT; ++q) {
            ok[q] = (j0 + q * ncons) < p.packs;
#pragma unroll
            for (int e = 0; e < 8; ++e) y[q][e] = 0.f;
          }
          for (int k = 0; k < nseg; ++k) {
            if (k > 0 && !*abort_flag && !mbar_wait(&full[slot], phase, abort_flag, p.wait_limit_ns)) {
              if (!*abort_flag) atomicOr(&g_far_error, kErrWaitFull);
              *abort_flag = 1;
            }
            const uint4* seg = reinterpret_cast<const uint4*>(ring + static_cast<size_t>(slot) * seg_bytes);
#pragma unroll
            for (int q = 0; q < VPT; ++q)
              if (ok[q]) add_pack<DT>(seg[j0 + q * ncons], y[q]);  // 0 + x: exact widening
            __syncwarp();
            if ((threadIdx.x & 31) == 0) mbar_arrive(&empty[slot]);
            if (++slot == nslot) {
              slot = 0;
              phase ^= 1u;
            }
          }
          const int64_t rbase = row * static_cast<int64_t>(p.packs);
          const float rinv = fabsf(w);
          if constexpr (MODE == kModeTensorNorm) {
            // the slot held norm_out round(o), or the row was rebuilt (y):
            // o itself is coded through gamma 1, weight_bias 0, rinv 1
            const float wb_ = rebuild ? p.weight_bias : 0.f;
            const float rinv_ = rebuild ? rinv : 1.f;
#pragma unroll
            for (int q = 0; q < VPT; ++q) {
              if (!ok[q]) continue;
              const int64_t pk = rbase + j0 + q * ncons;
              if (rebuild && p.residual_out != nullptr) static_cast<uint4*>(p.residual_out)[pk] = pack8<DT>(y[q]);
              const uint4 gm = rebuild ? gamma_pack(p, gamma_s, j0 + q * ncons) : ones_pack<DT>();
              reinterpret_cast<uint2*>(p.quant_out)[pk] =
                  tensor_codes<DT>(gm, wb_, y[q], rinv_, rinv_ * ts.inv, ts.scale, ts.inv, ts.exact);
            }
          } else {
            // the slot held the new residual round(y), or the row was rebuilt: y
#pragma unroll
            for (int q = 0; q < VPT; ++q) {
              if (!ok[q]) continue;
              const int64_t pk = rbase + j0 + q * ncons;
              if (rebuild) static_cast<uint4*>(p.residual_out)[pk] = pack8<DT>(y[q]);
              reinterpret_cast<uint2*>(p.quant_out)[pk] =
                  tensor_codes<DT>(gamma_pack(p, gamma_s, j0 + q * ncons), p.weight_bias, y[q], rinv,
                                   rinv * ts.inv, ts.scale, ts.inv, ts.exact);
            }
          }
        }
      }
    }
  }

  // Only after an abort can copies still be in flight: thread 0 waits for
  // the producer to stop and then for the last phase of every used slot.
  if (threadIdx.x == 0) {
    const uint64_t t0 = global_ns();
    while (!*producer_done && global_ns() - t0 < p.wait_limit_ns) {
    }
    if (*abort_flag) {
      const int64_t issued = *issued_count;
      for (int64_t g = (issued > nslot ? issued - nslot : 0); g < issued; ++g) {
        const int slot = static_cast<int>(g % nslot);
        mbar_wait(&full[slot], static_cast<uint32_t>(g / nslot) & 1u, nullptr, p.wait_limit_ns);
      }
    }
  }
}

// Second pass of dynamic per-tensor FP8 after a first pass that stored the
// new residual (no norm_out is written): each row's o is formed from its
// new residual round(y), read back from residual_out, as
// o = (round(y) * rinv) * (gamma + weight_bias) with the first pass's rinv,
// and only the codes are written: 3 bytes per element instead of a second
// read of every input.  round(y) is y to within half an ulp of the 2-byte
// format; below the format's normal range it is exact (every fp32 partial
// sum of 2-byte inputs is a whole multiple of the format's smallest
// subnormal), so a code differs by at most one step from the code of o
// formed from y itself.  A row the first pass flagged (sign bit of its
// stored rinv: an element may round to infinity) has no stored residual:
// its y is rebuilt from the partials and the residual in the first pass's
// order (the same bits), and its new residual is written here.
// blockDim = (tpr, rows_per_cta); rows in grid-stride order.
// kRows rows per thread per iteration (both rows' loads in flight before
// either is converted); measured on the W=4 8192 x 8192 call, two rows gave
// 179-180 us per call against 178 us with one, so one it is.
template <class DT, int VPT>
__global__ void __launch_bounds__(kMaxThreads)
far_tensor_quant_kernel(const Params p) {
  constexpr int kRows = 1;
  pdl_enter();
  const int64_t nrows = p.row_end - p.row_begin;
  const TensorScale ts(p, *p.ws_amax);
  const float scale = ts.scale, inv = ts.inv;
  const bool exact = ts.exact;
  const int j0 = threadIdx.x, tpr = blockDim.x;
  const uint4* gamma = static_cast<const uint4*>(p.gamma);
  const uint64_t drop = l2_evict_first();
  bool ok[VPT];
#pragma unroll
  for (int q = 0; q < VPT; ++q) ok[q] = j0 + q * tpr < p.packs;
  const int64_t step = static_cast<int64_t>(gridDim.x) * blockDim.y;
  for (int64_t k = static_cast<int64_t>(blockIdx.x) * blockDim.y + threadIdx.y; k < nrows;
       k += kRows * step) {
    const bool two = kRows == 2 && k + step < nrows;
    const int64_t ra = call_row(p, k);
    const int64_t rb = two ? call_row(p, k + step) : ra;
    const float wa = p.ws_rinv[ra - p.ws_row0];
    const float wb = two ? p.ws_rinv[rb - p.ws_row0] : 0.f;
    if (signbit(wa) || signbit(wb)) {  // a row to rebuild: each row on its own
      tensor_quant_row<DT, VPT>(p, ra, wa, j0, tpr, ok, inv, scale, exact, drop);
      if (two) tensor_quant_row<DT, VPT>(p, rb, wb, j0, tpr, ok, inv, scale, exact, drop);
      continue;
    }
    const int64_t ba = ra * static_cast<int64_t>(p.packs), bb = rb * static_cast<int64_t>(p.packs);
    const uint4* src = static_cast<const uint4*>(p.tensor_source == 2 ? p.norm_out : p.residual_out);
    uint4 va[VPT], vb[VPT], gv[VPT];
#pragma unroll
    for (int q = 0; q < VPT; ++q) {
      va[q] = vb[q] = gv[q] = make_uint4(0u, 0u, 0u, 0u);
      if (ok[q]) {
        va[q] = ld_once_l2_hint(src + ba + j0 + q * tpr, drop);
        if (two) vb[q] = ld_once_l2_hint(src + bb + j0 + q * tpr, drop);
        if (p.tensor_source == 1) gv[q] = __ldg(gamma + j0 + q * tpr);
      }
    }
    const float rinv_a = fabsf(wa), rinv_b = fabsf(wb);
#pragma unroll
    for (int q = 0; q < VPT; ++q) {
      if (!ok[q]) continue;
      reinterpret_cast<uint2*>(p.quant_out)[ba + j0 + q * tpr] = stored_codes<DT>(
          p.tensor_source, va[q], gv[q], p.weight_bias, rinv_a, rinv_a * inv, scale, inv, exact);
    }
    if (two) {
#pragma unroll
      for (int q = 0; q < VPT; ++q) {
        if (!ok[q]) continue;
        reinterpret_cast<uint2*>(p.quant_out)[bb + j0 + q * tpr] = stored_codes<DT>(
            p.tensor_source, vb[q], gv[q], p.weight_bias, rinv_b, rinv_b * inv, scale, inv, exact);
      }
    }
  }
}

// Launch attributes: programmatic stream serialization (PDL) and a cluster
// shape.
struct Attrs {
  cudaLaunchAttribute a[2];
  unsigned n = 0;
  Attrs(const Launch& l, int cluster) {
    if (l.pdl) {
      a[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      a[n].val.programmaticStreamSerializationAllowed = 1;
      ++n;
    }
    if (cluster > 0) {
      a[n].id = cudaLaunchAttributeClusterDimension;
      a[n].val.clusterDim.x = static_cast<unsigned>(cluster);
      a[n].val.clusterDim.y = 1;
      a[n].val.clusterDim.z = 1;
      ++n;
    }
  }
};

template <class DT, int VPT, bool SUB, int MODE>
cudaError_t launch_prefill_t(const Params& p, const Launch& l, cudaStream_t s) {
  Attrs at(l, 0);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(l.grid), 1, 1);
  cfg.blockDim = dim3(static_cast<unsigned>(l.tpr), static_cast<unsigned>(l.rows_per_cta), 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cfg.attrs = at.a;
  cfg.numAttrs = at.n;
  return cudaLaunchKernelEx(&cfg, far_prefill_kernel<DT, VPT, SUB, MODE>, p);
}

template <class DT, int VPT>
cudaError_t launch_decode_t(const Params& p, const Launch& l, cudaStream_t s) {
  Attrs at(l, l.cluster);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(l.cluster), static_cast<unsigned>(l.grid / l.cluster), 1);
  cfg.blockDim = dim3(static_cast<unsigned>(l.threads), 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cfg.attrs = at.a;
  cfg.numAttrs = at.n;
  return cudaLaunchKernelEx(&cfg, far_decode_kernel<DT, VPT>, p);
}

template <class DT, int VPT, int MINB, int MODE, int MAXC = kRingMaxConsumers>
cudaError_t launch_ring_t(const Params& p, const Launch& l, cudaStream_t s) {
  Attrs at(l, 0);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(l.grid), 1, 1);
  cfg.blockDim = dim3(static_cast<unsigned>(l.threads), 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(l.smem_bytes);
  cfg.stream = s;
  cfg.attrs = at.a;
  cfg.numAttrs = at.n;
  return cudaLaunchKernelEx(&cfg, far_ring_kernel<DT, VPT, MINB, MODE, MAXC>, p, l.nslot, l.tpr,
                            l.ring_gamma);
}

template <class DT, int MODE>
cudaError_t launch_ring_g(const Params& p, const Launch& l, cudaStream_t s) {
  const bool three = l.ring_minb >= 3;
  switch (l.vpt) {
    case 1: return three ? launch_ring_t<DT, 1, 3, MODE>(p, l, s) : launch_ring_t<DT, 1, 2, MODE>(p, l, s);
    case 2:
      if constexpr (MODE != kModeGroup)
        if (l.ring_wide) return launch_ring_t<DT, 2, 2, MODE, kRingWide2Consumers>(p, l, s);
      return three ? launch_ring_t<DT, 2, 3, MODE>(p, l, s) : launch_ring_t<DT, 2, 2, MODE>(p, l, s);
    case 4:
      if (l.ring_wide)
        return l.ring_minb == 1 ? launch_ring_t<DT, 4, 1, MODE, kRingWide1Consumers>(p, l, s)
                                : launch_ring_t<DT, 4, 2, MODE, kRingWideConsumers>(p, l, s);
      return three ? launch_ring_t<DT, 4, 3, MODE>(p, l, s) : launch_ring_t<DT, 4, 2, MODE>(p, l, s);
    case 8: return l.ring_minb >= 2 ? launch_ring_t<DT, 8, 2, MODE>(p, l, s)
                                    : launch_ring_t<DT, 8, 1, MODE>(p, l, s);
    default: return cudaErrorInvalidConfiguration;
  }
}

template <class DT>
cudaError_t launch_ring_dt(const Params& p, const Launch& l, cudaStream_t s) {
  switch (mode_of(p.pattern)) {
    case kModeGroup: return launch_ring_g<DT, kModeGroup>(p, l, s);
    case kModeTensor:
      return p.tensor_source == 2 ? launch_ring_g<DT, kModeTensorNorm>(p, l, s)
                                  : launch_ring_g<DT, kModeTensor>(p, l, s);
    default: return launch_ring_g<DT, kModePlain>(p, l, s);
  }
}

template <class DT, int MODE>
cudaError_t launch_prefill_g(const Params& p, const Launch& l, cudaStream_t s) {
  if (l.tpr <= 32 && l.rows_per_cta > 1) return launch_prefill_t<DT, 1, true, MODE>(p, l, s);
  switch (l.vpt) {
    case 1: return launch_prefill_t<DT, 1, false, MODE>(p, l, s);
    case 2: return launch_prefill_t<DT, 2, false, MODE>(p, l, s);
    case 4: return launch_prefill_t<DT, 4, false, MODE>(p, l, s);
    case 8: return launch_prefill_t<DT, 8, false, MODE>(p, l, s);
    default: return cudaErrorInvalidConfiguration;
  }
}

template <class DT>
cudaError_t launch_prefill_dt(const Params& p, const Launch& l, cudaStream_t s) {
  switch (mode_of(p.pattern)) {
    case kModeGroup: return launch_prefill_g<DT, kModeGroup>(p, l, s);
    case kModeTensor:
      return p.tensor_source == 2 ? launch_prefill_g<DT, kModeTensorNorm>(p, l, s)
                                  : launch_prefill_g<DT, kModeTensor>(p, l, s);
    default: return launch_prefill_g<DT, kModePlain>(p, l, s);
  }
}

template <class DT, int VPT>
cudaError_t launch_tensor_quant_t(const Params& p, const Launch& l, cudaStream_t s) {
  Attrs at(l, 0);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(l.grid), 1, 1);
  cfg.blockDim = dim3(static_cast<unsigned>(l.tpr), static_cast<unsigned>(l.rows_per_cta), 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cfg.attrs = at.a;
  cfg.numAttrs = at.n;
  return cudaLaunchKernelEx(&cfg, far_tensor_quant_kernel<DT, VPT>, p);
}

template <class DT>
cudaError_t launch_tensor_quant_dt(const Params& p, const Launch& l, cudaStream_t s) {
  switch (l.vpt) {
    case 1: return launch_tensor_quant_t<DT, 1>(p, l, s);
    case 2: return launch_tensor_quant_t<DT, 2>(p, l, s);
    case 4: return launch_tensor_quant_t<DT, 4>(p, l, s);
    case 8: return launch_tensor_quant_t<DT, 8>(p, l, s);
    default: return cudaErrorInvalidConfiguration;
  }
}

template <class DT>
cudaError_t launch_decode_dt(const Params& p, const Launch& l, cudaStream_t s) {
  switch (l.vpt) {
    case 1: return launch_decode_t<DT, 1>(p, l, s);
    case 2: return launch_decode_t<DT, 2>(p, l, s);
    case 4: return launch_decode_t<DT, 4>(p, l, s);
    case 8: return launch_decode_t<DT, 8>(p, l, s);
    default: return cudaErrorInvalidConfiguration;
  }
}

template <class DT>
cudaError_t allow_large_smem() {
  cudaError_t e = cudaSuccess;
  const auto set = [&](auto kern) {
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kRingSmemMax);
  };
  set(far_ring_kernel<DT, 1, 2, kModePlain>);
  set(far_ring_kernel<DT, 2, 2, kModePlain>);
  set(far_ring_kernel<DT, 4, 2, kModePlain>);
  set(far_ring_kernel<DT, 1, 3, kModePlain>);
  set(far_ring_kernel<DT, 2, 3, kModePlain>);
  set(far_ring_kernel<DT, 4, 3, kModePlain>);
  set(far_ring_kernel<DT, 8, 1, kModePlain>);
  set(far_ring_kernel<DT, 8, 2, kModePlain>);
  set(far_ring_kernel<DT, 1, 2, kModeGroup>);
  set(far_ring_kernel<DT, 2, 2, kModeGroup>);
  set(far_ring_kernel<DT, 4, 2, kModeGroup>);
  set(far_ring_kernel<DT, 1, 3, kModeGroup>);
  set(far_ring_kernel<DT, 2, 3, kModeGroup>);
  set(far_ring_kernel<DT, 4, 3, kModeGroup>);
  set(far_ring_kernel<DT, 8, 1, kModeGroup>);
  set(far_ring_kernel<DT, 8, 2, kModeGroup>);
  set(far_ring_kernel<DT, 1, 2, kModeTensor>);
  set(far_ring_kernel<DT, 2, 2, kModeTensor>);
  set(far_ring_kernel<DT, 4, 2, kModeTensor>);
  set(far_ring_kernel<DT, 1, 3, kModeTensor>);
  set(far_ring_kernel<DT, 2, 3, kModeTensor>);
  set(far_ring_kernel<DT, 4, 3, kModeTensor>);
  set(far_ring_kernel<DT, 8, 1, kModeTensor>);
  set(far_ring_kernel<DT, 8, 2, kModeTensor>);
  set(far_ring_kernel<DT, 4, 2, kModePlain, kRingWideConsumers>);
  set(far_ring_kernel<DT, 4, 2, kModeTensor, kRingWideConsumers>);
  set(far_ring_kernel<DT, 2, 2, kModePlain, kRingWide2Consumers>);
  set(far_ring_kernel<DT, 2, 2, kModeTensor, kRingWide2Consumers>);
  set(far_ring_kernel<DT, 4, 1, kModePlain, kRingWide1Consumers>);
  set(far_ring_kernel<DT, 4, 1, kModeTensor, kRingWide1Consumers>);
  set(far_ring_kernel<DT, 1, 2, kModeTensorNorm>);
  set(far_ring_kernel<DT, 2, 2, kModeTensorNorm>);
  set(far_ring_kernel<DT, 4, 2, kModeTensorNorm>);
  set(far_ring_kernel<DT, 1, 3, kModeTensorNorm>);
  set(far_ring_kernel<DT, 2, 3, kModeTensorNorm>);
  set(far_ring_kernel<DT, 4, 3, kModeTensorNorm>);
  set(far_ring_kernel<DT, 8, 1, kModeTensorNorm>);
  set(far_ring_kernel<DT, 8, 2, kModeTensorNorm>);
  set(far_ring_kernel<DT, 4, 2, kModeTensorNorm, kRingWideConsumers>);
  set(far_ring_kernel<DT, 2, 2, kModeTensorNorm, kRingWide2Consumers>);
  set(far_ring_kernel<DT, 4, 1, kModeTensorNorm, kRingWide1Consumers>);
  set(far_ring_kernel<DT, 4, 2, kModeGroup, kRingWideConsumers>);
  set(far_ring_kernel<DT, 4, 1, kModeGroup, kRingWide1Consumers>);
  return e;
}

template <class DT>
cudaError_t allow_large_clusters() {
  cudaError_t e = cudaSuccess;
  const auto set = [&](auto kern) {
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  };
  set(far_decode_kernel<DT, 1>);
  set(far_decode_kernel<DT, 2>);
  set(far_decode_kernel<DT, 4>);
  set(far_decode_kernel<DT, 8>);
  return e;
}

}  // namespace

cudaError_t launch_prefill(const Params& p, int dtype, const Launch& l, cudaStream_t s) {
  return dtype == kBf16 ? launch_prefill_dt<Bf16T>(p, l, s) : launch_prefill_dt<Fp16T>(p, l, s);
}

cudaError_t launch_decode(const Params& p, int dtype, const Launch& l, cudaStream_t s) {
  return dtype == kBf16 ? launch_decode_dt<Bf16T>(p, l, s) : launch_decode_dt<Fp16T>(p, l, s);
}

cudaError_t launch_ring(const Params& p, int dtype, const Launch& l, cudaStream_t s) {
  return dtype == kBf16 ? launch_ring_dt<Bf16T>(p, l, s) : launch_ring_dt<Fp16T>(p, l, s);
}

cudaError_t launch_tensor_quant(const Params& p, int dtype, const Launch& l, cudaStream_t s) {
  return dtype == kBf16 ? launch_tensor_quant_dt<Bf16T>(p, l, s)
                        : launch_tensor_quant_dt<Fp16T>(p, l, s);
}

int ring_header_bytes(int nslot) { return ring_offset(nslot); }

namespace {
template <class DT, int VPT, int MINB, int MAXC = kRingMaxConsumers>
int occ_of(int threads, int smem) {
  // the per-group instantiation is sized the same way; the plain one decides
  int n = 0;
  const cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
      &n, far_ring_kernel<DT, VPT, MINB, kModePlain, MAXC>, threads, smem);
  return e == cudaSuccess ? n : 0;
}

template <class DT>
int ring_occupancy_dt(int vpt, int minb, int threads, int smem) {
  const bool three = minb >= 3;
  switch (vpt) {
    case 1: return three ? occ_of<DT, 1, 3>(threads, smem) : occ_of<DT, 1, 2>(threads, smem);
    case 2:
      if (threads > kRingMaxConsumers + 32) return occ_of<DT, 2, 2, kRingWide2Consumers>(threads, smem);
      return three ? occ_of<DT, 2, 3>(threads, smem) : occ_of<DT, 2, 2>(threads, smem);
    case 4:
      if (threads > kRingWideConsumers + 32) return occ_of<DT, 4, 1, kRingWide1Consumers>(threads, smem);
      if (threads > kRingMaxConsumers + 32) return occ_of<DT, 4, 2, kRingWideConsumers>(threads, smem);
      return three ? occ_of<DT, 4, 3>(threads, smem) : occ_of<DT, 4, 2>(threads, smem);
    case 8: return minb >= 2 ? occ_of<DT, 8, 2>(threads, smem) : occ_of<DT, 8, 1>(threads, smem);
    default: return 0;
  }
}
}  // namespace

int decode_occupancy(int dtype, int vpt, int threads) {
  int n = 0;
  cudaError_t e = cudaErrorInvalidValue;
  const auto occ = [&](auto kern) {
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, threads, 0);
  };
  const bool bf = dtype == kBf16;
  switch (vpt) {
    case 1: bf ? occ(far_decode_kernel<Bf16T, 1>) : occ(far_decode_kernel<Fp16T, 1>); break;
    case 2: bf ? occ(far_decode_kernel<Bf16T, 2>) : occ(far_decode_kernel<Fp16T, 2>); break;
    case 4: bf ? occ(far_decode_kernel<Bf16T, 4>) : occ(far_decode_kernel<Fp16T, 4>); break;
    case 8: bf ? occ(far_decode_kernel<Bf16T, 8>) : occ(far_decode_kernel<Fp16T, 8>); break;
    default: return 0;
  }
  return e == cudaSuccess ? n : 0;
}

int ring_occupancy(int dtype, int vpt, int minb, int threads, int smem_bytes) {
  return dtype == kBf16 ? ring_occupancy_dt<Bf16T>(vpt, minb, threads, smem_bytes)
                        : ring_occupancy_dt<Fp16T>(vpt, minb, threads, smem_bytes);
}

cudaError_t configure_kernels() {
  cudaError_t e = allow_large_clusters<Bf16T>();
  if (e == cudaSuccess) e = allow_large_clusters<Fp16T>();
  if (e == cudaSuccess) e = allow_large_smem<Bf16T>();
  if (e == cudaSuccess) e = allow_large_smem<Fp16T>();
  return e;
}

cudaError_t read_error_word(unsigned* out, cudaStream_t s) {
  cudaError_t e = cudaMemcpyFromSymbolAsync(out, g_far_error, sizeof(unsigned), 0,
                                            cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  return e;
}

cudaError_t clear_error_word(cudaStream_t s) {
  static const unsigned zero = 0u;
  cudaError_t e = cudaMemcpyToSymbolAsync(g_far_error, &zero, sizeof(unsigned), 0,
                                          cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  return e;
}

// The per-tensor workspace header (amax, rows done, rows taken) set to zero
// by a kernel rather than a memset, so that the ring kernel after it can be
// launched with programmatic dependent launch: its set-up overlaps this one.
__global__ void far_ws_zero_kernel(unsigned* ws) {
  pdl_enter();  // the previous call's kernels have finished with the header
  if (threadIdx.x < 4) ws[threadIdx.x] = 0u;
}

cudaError_t launch_ws_zero(unsigned* ws, int pdl, cudaStream_t s) {
  cudaLaunchAttribute a[1];
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1, 1, 1);
  cfg.blockDim = dim3(32, 1, 1);
  cfg.stream = s;
  if (pdl) {
    a[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    a[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = a;
    cfg.numAttrs = 1;
  }
  return cudaLaunchKernelEx(&cfg, far_ws_zero_kernel, ws);
}
}  // namespace far

// far_abi.cu -- the C ABI declared in include/far.h: context, host-side
// argument checks, the choice between the decode and prefill launch shapes,
// and the launch.  No allocation, no synchronisation.
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>

#include <cuda_runtime.h>

#include "far.h"
#include "far_internal.h"

struct far_ctx {
  int device;
  int sm_count;
  int cc_major;
  int cc_minor;
  int decode_max_rows;  // rows <= this take the decode (cluster) kernel
  int force_regime;     // FAR_REGIME_*
  int decode_cluster;   // preferred CTAs per row in decode
  int prefill_threads;  // target threads per row in prefill
  int prefill_kernel;   // 1 = TMA bulk-copy ring (default), 0 = direct loads
  int ring_ctas_per_sm; // persistent ring CTAs per SM wanted (1..4; 0 = by rule)
  int ring_threads;     // target consumer threads of a ring CTA
  int ring_threads_set; // ring_threads came from the environment
  int ring_slots_max;   // at most this many ring slots
  int tensor_reverse;   // per-tensor FP8: second pass from the last row down
  int tensor_fused;     // per-tensor FP8: both passes in one ring launch when possible
  int ring_gamma_mode;
  int ring_wide;        // the wide ring build for rows of 1025-1536 packs (1 / 0)
  int ring_wide2;       // the wide 2-pack build for rows of 513-896 packs (1 / 0)
  int ring_wide1;       // the one-CTA wide build for rows of 1537-2048 packs (1 / 0)
  int ring_wide_group;  // per-group FP8 also takes the 384- and 512-consumer builds (1 / 0)  // ring: 1 stage gamma in shared memory, 0 read it through L1, -1 by rule
  int pdl;              // programmatic dependent launch on every call
  int ring_min_rows;    // fewer rows than this take the direct kernel
  uint64_t wait_limit_ns;  // bounded waits in the kernels give up after this
  int64_t stall_segment;   // test hook (far_test_stall), -1 when off
  // ring CTAs per SM the occupancy calculator allows, per (dtype, packs):
  // 0 = not asked yet, -1 = cannot run
  // resident ring CTAs per SM for the configurations asked so far
  struct OccEntry {
    int dtype, vpt, minb, threads, smem, ctas;
  };
  static constexpr int kOccEntries = 256;
  std::mutex occ_mu;
  OccEntry occ[kOccEntries];
  int occ_n;
  // far_fused_host: its two copy streams and the events of its two staging
  // buffers, created on first use, guarded by host_mu
  std::mutex host_mu;
  bool host_ready;
  cudaStream_t host_h2d, host_d2h;
  cudaEvent_t host_start, host_in[2], host_comp[2], host_out[2];
};

namespace {

thread_local char g_last_error[256] = "";

far_status cuda_fail(cudaError_t e, const char* what) {
  std::snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%s)", what,
                cudaGetErrorString(e), cudaGetErrorName(e));
  return FAR_ERR_CUDA;
}

int env_int(const char* name, int dflt) {
  const char* s = std::getenv(name);
  if (s == nullptr || *s == '\0') return dflt;
  char* end = nullptr;
  long v = std::strtol(s, &end, 10);
  return (end != s) ? static_cast<int>(v) : dflt;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Free far_fused_host's streams and events (each once its work is done).
void host_pipe_release(far_ctx* ctx) {
  if (!ctx->host_ready) return;
  int prev = -1;
  const bool switched = cudaGetDevice(&prev) == cudaSuccess && prev != ctx->device &&
                        cudaSetDevice(ctx->device) == cudaSuccess;
  cudaStreamDestroy(ctx->host_h2d);
  cudaStreamDestroy(ctx->host_d2h);
  cudaEventDestroy(ctx->host_start);
  for (int b = 0; b < 2; ++b) {
    cudaEventDestroy(ctx->host_in[b]);
    cudaEventDestroy(ctx->host_comp[b]);
    cudaEventDestroy(ctx->host_out[b]);
  }
  ctx->host_ready = false;
  if (switched) cudaSetDevice(prev);
}

struct Range {
  uintptr_t lo, hi;  // [lo, hi)
};

bool overlap(Range a, Range b) { return a.lo < b.hi && b.lo < a.hi; }

Range span(const void* p, int64_t bytes) {
  const uintptr_t lo = reinterpret_cast<uintptr_t>(p);
  return Range{lo, lo + static_cast<uintptr_t>(bytes)};
}

int pow2_floor(int x) {
  int p = 1;
  while (p * 2 <= x) p *= 2;
  return p;
}

int pow2_ceil(int x) {
  int p = 1;
  while (p < x) p *= 2;
  return p;
}

// Prefill geometry: the fewest packs per thread (1, 2, 4 or 8) that keep a
// row within `target` threads; rows of at most 32 packs share a CTA.
void plan_prefill(int packs, int target, far::Launch* l) {
  l->regime = FAR_REGIME_PREFILL;
  l->cluster = 1;
  if (packs <= 32) {
    l->vpt = 1;
    l->tpr = pow2_ceil(packs);
    l->rows_per_cta = far::kMaxThreads / l->tpr;
  } else {
    int vpt = 1;
    while (vpt < 8 && (packs + vpt - 1) / vpt > target) vpt *= 2;
    l->vpt = vpt;
    l->tpr = (((packs + vpt - 1) / vpt) + 31) / 32 * 32;
    l->rows_per_cta = 1;
  }
  l->threads = l->tpr * l->rows_per_cta;
}

// Decode geometry: `cluster` CTAs per row (a power of two, at most 16, and
// at most packs/32 so that each CTA has a warp of work, but large enough for
// the slice to fit 256 threads at up to 8 packs each), each CTA's slice held
// at 1, 2, 4 or 8 packs per thread.
void plan_decode(int packs, int cluster_pref, far::Launch* l) {
  l->regime = FAR_REGIME_DECODE;
  int cl = pow2_floor(cluster_pref < 1 ? 1 : (cluster_pref > 16 ? 16 : cluster_pref));
  while (cl > 1 && packs / cl < 32) cl /= 2;
  while (cl < 16 && (packs + cl - 1) / cl > 8 * far::kMaxThreads) cl *= 2;
  l->cluster = cl;
  const int chunk = (packs + cl - 1) / cl;
  int vpt = 1;
  while (vpt < 8 && (chunk + vpt - 1) / vpt > far::kMaxThreads) vpt *= 2;
  l->vpt = vpt;
  l->tpr = (((chunk + vpt - 1) / vpt) + 31) / 32 * 32;
  l->threads = l->tpr;
  l->rows_per_cta = 1;
}

// Resident ring CTAs per SM for one configuration, cached per context
// (the occupancy calculator costs microseconds): 0 = cannot run.
int ring_occ_cached(const far_ctx* ctx, int dtype, int vpt, int minb, int threads, int smem);

// Ring geometry.  Every rule was measured on B200 against its alternatives
// (fractions of the measured HBM copy bandwidth, static FP8, bf16, W = 2, 4
// and 8 at H = 2048-16384, about 768 MiB of inputs per call) and is used
// only where it won.
//
// Consumers: the fewest packs per thread (1, 2, 4, 8) that keep within
// ring_threads (256), plus one producer warp.  Two exceptions:
//  * rows of 512-1023 packs with at most 6 segments take 4 packs per
//    thread (H=4096, W=4: 128-thread CTAs, 97 vs 85 %);
//  * rows of at most 256 packs (H <= 2048) take at most 128 consumers.
//
// CTAs per SM and slots.  What pays is many CTAs (consumer warps to hide
// the per-row latency) with few row-segment slots each: about 96 KiB of
// slots per SM in all.  More slots in flight lost everywhere (W=8,
// H=3072: 4 slots 99.8 %, 6 slots 97.0, 8 slots 92.5, at 4 CTAs per SM).
// By row length (packs = H / 8), CTAs per SM x slots per CTA:
//  * <= 256 packs: 6 x 4, with norm_out 4 x 6 (W=2/4/8: 93-100 vs 78-97 %
//    for the previous 4 x 12);
//  * <= 384: 4 x 4, with norm_out 3 x 4 (94-100 vs 83-93 %);
//  * <= 512: 4 x 3, 3 x 4 when norm_out is written or the row has more
//    than 6 segments (92-101 vs 90-100 %);
//  * <= 640: 4 x 3 (4 x 4 for at most 3 segments), with norm_out 4 x 2
//    (90-99 vs 88-97 %);
//  * <= 768: 4 x 2, with norm_out 2 x 4 (95-97 vs 92-97 %);
//  * <= 896: 2 x 4, 3 x 3 for 4-6 segments, with norm_out 3 x 2 (92-98 vs
//    83-97 %);
//  * <= 1024 (4 packs per thread): 3 x 3 for 5 or 6 segments (W=4 + residual,
//    the c4 shape: 97.4 %), else 2 x 4 (W=2: 98.8 vs 84.0 %); with norm_out
//    and at most 6 segments of at least 16 KiB, 2 CTAs per SM with gamma
//    read through L1 and about 96 KiB of slots (W=3..5: 97-102 vs 87-94 %);
//  * 513-896 packs (H = 4104-7168) with 8 or more segments (W=8 + the
//    residual): the wide 2-pack build, 2 packs per thread over up to 448
//    consumers, 2 CTAs per SM, about 56 KiB of slots each (W=8 at H=4608,
//    5120, 6144, 7168: 98-101 vs 93-98 %, per-token H=7168: 99.4 vs 97.1 %;
//    at 3-5 segments it lost as often as it won);
//  * 1025-1536 packs (H = 8200-12288): the wide build, 4 packs per thread
//    over up to 384 consumers, 2 CTAs per SM, about 72 KiB of slots (W=2/
//    3/4/8 at H=10240: 94-97 vs 76-89 %; at H=12288: 86-98 vs 80-91 %);
//    for at most 4 segments gamma through L1 and a slot per segment (W=2
//    at H=10240 / 12288: 97.7 / 96.6 vs 94.6 / 84.1 %; W=3: 98.0 / 99.1
//    vs 95.8 / 98.1 %); with norm_out and at most 6 segments gamma through
//    L1 and 2 slots (W=2/3/4 at H=10240 / 12288: 92-97 vs 86-94 %, where
//    the default slots lost);
//  * 1537-2048 packs (H = 12296-16384) without norm_out, or with more than
//    6 segments: the one-CTA wide build, 4 packs per thread over up to 512
//    consumers, one CTA per SM, 6 slots, 4 for rows of at most 4 segments
//    (W=2/3/4/8 at H=16384: 88-98 vs 85-90 %; at H=14336: 88-97 vs
//    80-89 %; with norm_out and 3-5 segments it lost up to 9 points);
//  * 8 packs per thread (H >= 12288): 2 CTAs per SM, with the build whose
//    registers are sized for two, about 72 KiB of slots (H=12288, W=2..8:
//    80-93 vs 58-84 % at one CTA); but one CTA per SM with 6 slots when the
//    row has more than 6 segments and fewer than 3 slots fit the 2-CTA share
//    (H=16384, W=8: 87-90 %).
// Per-group FP8 (more work per row, and more registers) has a rule of its
// own, from sweeps of CTAs per SM x slots at H = 2048-12288, W = 2-8,
// with and without norm_out: up to 6 segments, 5 CTAs per SM x 6 slots up
// to 256 packs and 5 x 4 up to 512 (W=2-4 at H=2048 / 4096: 72-97 vs
// 65-90 % with 4 CTAs); 4 x 4 up to 640 (4 x 6 beyond 6 segments, and
// beyond 6 segments from 257 packs); 4 x 4 up to 768 (H=6144, W=2-4:
// 81-96 vs 69-90 % at 3 x 3); 3 x 3 up to 1024 (W=8 at H=4096 / 5120:
// 96-99 vs 79-90 %; with norm_out at H=4096 / 5120 / 8192, W=2-4: 83-95
// vs 63-87 %; the static rule lost for it: mean 86.5 against 90.3 % at
// W=4 / 8, H=4096 / 7168).  Beyond 1024 packs it takes the 384-
// and 512-consumer builds (the one-CTA build with norm_out too), whose
// registers do not spill as 8 packs per thread do (H = 10240-16384:
// 65-97 vs 49-81 %).
// Dynamic per-tensor FP8 (both passes in one launch, the second reading
// rows back from L2) wants more CTAs per SM below H = 4096 and fewer slots:
// its own rule from H = 2048 to 4096 and at H = 8192, the static rule
// elsewhere.
// Gamma is staged in shared memory unless said otherwise; where the slots
// asked for do not fit, as many as fit; below 2 (below 3 for the byte
// targets), the rule falls back to 2 CTAs per SM with gamma through L1.
//
// Environment overrides (FAR_RING_CTAS_PER_SM, FAR_RING_THREADS,
// FAR_RING_SLOTS, FAR_RING_GAMMA_SMEM) replace the rule they name.  The grid
// is persistent: sm_count x (the CTAs per SM the occupancy calculator
// confirms), fewer for fewer rows.  Returns false (the direct kernel runs)
// when fewer than two slots fit or the configuration cannot be resident.
bool plan_ring(const far_ctx* ctx, int packs, int64_t rows, int dtype, int segs, bool norm,
               bool group, bool tensor, far::Launch* l) {
  if (packs <= 32) return false;
  const int seg = packs * 16;
  const bool small_rows = packs <= 256;  // H <= 2048
  const int max_cons = !ctx->ring_threads_set && small_rows ? 128 : ctx->ring_threads;
  int vpt = 1;
  while (vpt < 8 && (packs + vpt - 1) / vpt > max_cons) vpt *= 2;
  if (!ctx->ring_threads_set && segs <= 6 && packs >= 512 && packs < 1024 && vpt < 4) vpt = 4;
  // rows of 1025-1536 packs: the wide build, 4 packs per thread over up to
  // 384 consumers, instead of 8 packs per thread
  const bool wide4 = ctx->ring_wide && !ctx->ring_threads_set && (!group || ctx->ring_wide_group) &&
                     packs > 1024 && packs <= 4 * far::kRingWideConsumers;
  // rows of 513-896 packs with 8 or more segments: 2 packs per thread over
  // up to 448 consumers
  const bool wide2 = ctx->ring_wide2 && !ctx->ring_threads_set && !group && packs > 512 &&
                     packs <= 2 * far::kRingWide2Consumers && segs >= 8;
  // rows of 1537-2048 packs without norm_out (or with more than 6
  // segments): one CTA per SM of up to 512 consumers, 4 packs each
  const bool wide1 = ctx->ring_wide1 && !ctx->ring_threads_set && (!group || ctx->ring_wide_group) &&
                     packs > 1536 && packs <= 4 * far::kRingWide1Consumers &&
                     (!norm || segs > 6 || group);
  const bool wide = wide4 || wide2 || wide1;
  if (wide4 || wide1) vpt = 4;
  if (wide2) vpt = 2;
  const int tpr = (((packs + vpt - 1) / vpt) + 31) / 32 * 32;
  if (tpr > (wide1 ? far::kRingWide1Consumers : wide4 ? far::kRingWideConsumers
                                              : wide2 ? far::kRingWide2Consumers
                                                      : far::kRingMaxConsumers))
    return false;

  int n_req = 2;
  bool gamma_smem = true;
  int want = 0;            // slots per CTA (0: by `target` bytes)
  int target = 72 * 1024;  // slot bytes per CTA when want == 0
  if (wide1) {
    // one CTA per SM; 4 slots for rows of at most 4 segments without
    // norm_out (W=2/3 at H=14336 / 16384: 88-98 vs 85-95 % with 6), else 6
    n_req = 1;
    want = (!norm && segs <= 4) ? 4 : 6;
  } else if (wide4) {
    // 2 CTAs per SM (its registers are sized for two), about 72 KiB of
    // slots; for rows of at most 4 segments gamma through L1 and one slot
    // per segment; with norm_out and at most 6 segments gamma through L1
    // and 2 slots
    if (norm && segs <= 6) {
      gamma_smem = false;
      want = 2;
    } else if (segs <= 4) {
      gamma_smem = false;
      want = segs < 3 ? 3 : segs;
    }
  } else if (wide2) {
    // 2 CTAs per SM, about 56 KiB of slots each
    want = 56 * 1024 / seg;
    if (want < 2) want = 2;
  } else if (vpt >= 8) {
    // 8 packs per thread: 2 CTAs per SM (a build with a few spilled
    // registers), unless the row has many segments and fewer than 3 slots
    // would fit: then one CTA per SM, as all its registers allow, 6 slots
    if (segs > 6 && ctx->ring_slots_max == 0 &&
        (228 * 1024 / 2 - 1024 - 1024) / seg - 1 < 3) {
      n_req = 1;
      target = 6 * seg;
    }
  } else if (group) {
    // per-group FP8 (more work per row), measured on its own
    if (packs <= 512 && segs <= 6) {
      n_req = 5;
      want = packs <= 256 ? 6 : 4;
    } else if (packs <= 640) {
      n_req = 4;
      want = segs > 6 ? 6 : 4;
    } else if (packs <= 768) {
      n_req = 4;
      want = 4;
    } else {
      n_req = 3;
      want = 3;
    }
  } else if (tensor && packs > 256 && packs <= 384 && norm) {
    // dynamic per-tensor FP8 (two passes in one launch) has a rule of its
    // own, from sweeps of CTAs per SM x slots at H = 2048-8192, W = 2-8:
    // H = 2056-3072 with norm_out 4 x 6 (W=2/3/4/8: 75-86 vs 65-79 %)
    n_req = 4;
    want = 6;
  } else if (tensor && (packs <= 256 || (packs <= 512 && segs <= 6))) {
    // ... H <= 2048 6 x 4, with norm_out too (W=2/3/4/8 with norm_out:
    // 72-85 vs 62-80 %); H <= 4096 with at most 6 segments 5 x 4 (W=2/3/4
    // at H=4096: 75-83 vs 65-78 %)
    n_req = packs <= 256 ? 6 : 5;
    want = 4;
  } else if (tensor && packs > 896 && packs <= 1024) {
    // ... H=8192: 3 x 3 for every W, with norm_out too (W=2/3/4: 78-85 vs
    // 71-82 %)
    n_req = 3;
    want = 3;
  } else if (packs <= 256) {
    n_req = norm ? 4 : 6;
    want = norm ? 6 : 4;
  } else if (packs <= 384) {
    n_req = norm ? 3 : 4;
    want = 4;
  } else if (packs <= 512) {
    n_req = (norm || segs > 6) ? 3 : 4;
    want = (norm || segs > 6) ? 4 : 3;
  } else if (packs <= 640) {
    n_req = 4;
    want = norm ? 2 : (segs <= 3 ? 4 : 3);
  } else if (packs <= 768) {
    n_req = norm ? 2 : 4;
    want = norm ? 4 : 2;
  } else if (packs <= 896) {
    const bool mid = !norm && segs >= 4 && segs <= 6;
    n_req = norm || mid ? 3 : 2;
    want = norm ? 2 : (mid ? 3 : 4);
  } else if (norm && segs <= 6 && seg >= 16 * 1024) {
    gamma_smem = false;
    target = 96 * 1024;
  } else if (segs == 5 || segs == 6) {
    n_req = 3;
    want = 3;
  } else {
    want = 4;
  }
  if (ctx->ring_ctas_per_sm > 0) n_req = ctx->ring_ctas_per_sm;
  if (ctx->ring_gamma_mode >= 0) gamma_smem = ctx->ring_gamma_mode != 0;
  auto fit = [&](int n, bool gs, int bytes, int slots) {
    int per_cta = 228 * 1024 / n - 1024;
    if (per_cta > far::kRingSmemMax) per_cta = far::kRingSmemMax;
    int ns = ctx->ring_slots_max > 0 ? ctx->ring_slots_max : (slots > 0 ? slots : bytes / seg);
    if (ns > 32) ns = 32;
    while (ns >= 2 && far::ring_header_bytes(ns) + (ns + (gs ? 1 : 0)) * seg > per_cta) --ns;
    return ns;
  };
  int nslot = fit(n_req, gamma_smem, target, want);
  if (nslot < (want > 0 ? 2 : 3) && vpt < 8 && ctx->ring_ctas_per_sm == 0 && ctx->ring_gamma_mode < 0) {
    n_req = 2;
    gamma_smem = false;
    nslot = fit(n_req, gamma_smem, 96 * 1024, 0);
  }
  if (nslot < 2) return false;
  const int gsegs = gamma_smem ? 1 : 0;
  const int smem = far::ring_header_bytes(nslot) + (nslot + gsegs) * seg;
  // the register budget the kernel is built for: 3 or 2 CTAs per SM, and at
  // 8 packs per thread 1 (no spills) or 2 (a few spilled registers)
  const int minb = wide1 ? 1 : wide ? 2 : vpt >= 8 ? (n_req >= 2 ? 2 : 1) : (n_req >= 3 ? 3 : 2);
  int occ = ring_occ_cached(ctx, dtype, vpt, minb, tpr + 32, smem);
  if (occ < 1) return false;
  if (occ > n_req) occ = n_req;
  l->kernel = 1;
  l->ring_minb = minb;
  l->ring_gamma = gsegs;
  l->ring_wide = wide ? 1 : 0;
  l->vpt = vpt;
  l->tpr = tpr;
  l->rows_per_cta = 1;
  l->nslot = nslot;
  l->smem_bytes = smem;
  l->threads = tpr + 32;
  const int64_t ctas = static_cast<int64_t>(ctx->sm_count) * occ;
  l->grid = rows < ctas ? rows : ctas;
  return true;
}

int ring_occ_cached(const far_ctx* ctx, int dtype, int vpt, int minb, int threads, int smem) {
  far_ctx* c = const_cast<far_ctx*>(ctx);
  std::lock_guard<std::mutex> lock(c->occ_mu);
  for (int i = 0; i < c->occ_n; ++i) {
    const far_ctx::OccEntry& e = c->occ[i];
    if (e.dtype == dtype && e.vpt == vpt && e.minb == minb && e.threads == threads && e.smem == smem)
      return e.ctas;
  }
  // minb < 0 marks the decode kernel's entries
  const int n = minb < 0 ? far::decode_occupancy(dtype, vpt, threads)
                         : far::ring_occupancy(dtype, vpt, minb, threads, smem);
  if (c->occ_n < far_ctx::kOccEntries) c->occ[c->occ_n++] = far_ctx::OccEntry{dtype, vpt, minb, threads, smem, n};
  return n;
}

// segs = row segments read per row: W partials, plus the residual if any;
// norm: the call writes norm_out.
far::Launch plan(const far_ctx* ctx, int64_t rows, int64_t H, int dtype, int segs, bool norm,
                 bool group = false, bool tensor = false) {
  const int packs = static_cast<int>(H / far::kPackElems);
  far::Launch l{};
  bool decode;
  if (ctx->force_regime == FAR_REGIME_DECODE) {
    decode = true;
  } else if (ctx->force_regime == FAR_REGIME_PREFILL) {
    decode = false;
  } else {
    // Measured on B200 with inputs cold in L2 (CUDA graphs cycling through
    // more than 2x L2), rows <= 80: a cluster per row beats one CTA per row
    // once that CTA would need 4 or more packs per thread (H >= 8192 at 256
    // threads: 2.8-4.1 vs 3.6-4.2 us at W=2, H=8192; 2.9-5.9 vs 6.2-7.6 us
    // at H=16384) or 32 or more loads per thread; at H=4096 the single
    // CTA's shorter path wins (W=2 and W=8: 2.4-3.9 vs 2.8-4.2 us).
    far::Launch d{};
    plan_prefill(packs, ctx->prefill_threads, &d);
    decode = rows <= ctx->decode_max_rows && packs >= 64 && (d.vpt >= 4 || segs * d.vpt >= 32);
  }
  if (decode) {
    int cl = ctx->decode_cluster;
    if (cl <= 0) {
      // measured (cold, as above): 16 CTAs per row for up to 4 rows, 8 up
      // to 16 rows, 4 beyond (T = 1 / 8 / 32 / 80 at H = 8192 and 16384)
      cl = rows <= 4 ? 16 : (rows <= 16 ? 8 : 4);
    }
    plan_decode(packs, cl, &l);
    // ... and no more CTAs than are resident in one wave: a second wave
    // costs more than a smaller cluster (H=16384, W=2, 80 rows: 4 CTAs per
    // row in two waves 7.6 us, 2 per row 5.9 us)
    if (ctx->decode_cluster <= 0) {
      while (l.cluster > 1) {
        const int occ = ring_occ_cached(ctx, dtype, l.vpt, -1, l.threads, 0);
        if (rows * l.cluster <= static_cast<int64_t>(occ) * ctx->sm_count) break;
        plan_decode(packs, l.cluster / 2, &l);
      }
    }
    l.grid = rows * l.cluster;
  } else {
    // The threads per row do not depend on the number of rows, so that row
    // slices of a call reduce each row in the same order as the whole call
    // (rows of 3 segments ran faster cold at 4 packs per thread from 4 rows
    // per SM up, W=2: 5.9 vs 6.4 us at 1024 x 2048, but a slice below that
    // size would then round differently from the whole call).
    plan_prefill(packs, ctx->prefill_threads, &l);
    l.grid = (rows + l.rows_per_cta - 1) / l.rows_per_cta;
    // The ring pays off once each persistent CTA gets enough rows to keep
    // its pipeline full: measured crossover about 8 rows per CTA at
    // H >= 7168 and 16 at H = 2048, i.e. max(8, 4096 / packs) per CTA.
    int64_t min_rows = ctx->ring_min_rows;
    if (min_rows <= 0) {
      const int per_cta = (4096 / packs > 8) ? 4096 / packs : 8;
      min_rows = static_cast<int64_t>(per_cta) * ctx->sm_count * 2;
    }
    if (ctx->prefill_kernel == 1 && rows >= min_rows) plan_ring(ctx, packs, rows, dtype, segs, norm, group, tensor, &l);
  }
  l.pdl = ctx->pdl;
  return l;
}

// The geometry a call of `pattern` runs with.  Per-group and per-tensor FP8
// plan the ring kernel by rules of their own and never take the cluster
// kernel: a group must sit on consecutive lanes of one warp, which a
// cluster CTA's slice need not start on, and the per-tensor second pass
// has no reduction for a cluster to share.
far::Launch plan_call(const far_ctx* ctx, int64_t rows, int64_t H, int dtype, int segs, bool norm,
                      int pattern) {
  const bool group = pattern == FAR_AR_RESIDUAL_RMSNORM_FP8_GROUP;
  const bool tensor = pattern == FAR_AR_RESIDUAL_RMSNORM_FP8_TENSOR;
  far::Launch l = plan(ctx, rows, H, dtype, segs, norm, group, tensor);
  if ((group || tensor) && l.regime == FAR_REGIME_DECODE) {
    plan_prefill(static_cast<int>(H / far::kPackElems), ctx->prefill_threads, &l);
    l.grid = (rows + l.rows_per_cta - 1) / l.rows_per_cta;
    l.pdl = ctx->pdl;
  }
  return l;
}

}  // namespace

extern "C" {

const char* far_status_string(far_status s) {
  switch (s) {
    case FAR_OK: return "FAR_OK";
    case FAR_ERR_INVALID_ARG: return "FAR_ERR_INVALID_ARG";
    case FAR_ERR_UNSUPPORTED: return "FAR_ERR_UNSUPPORTED";
    case FAR_ERR_ALIGNMENT: return "FAR_ERR_ALIGNMENT";
    case FAR_ERR_CUDA: return "FAR_ERR_CUDA";
    case FAR_ERR_TIMEOUT: return "FAR_ERR_TIMEOUT";
    case FAR_ERR_INTERNAL: return "FAR_ERR_INTERNAL";
  }
  return "FAR_ERR_UNKNOWN";
}

const char* far_last_error(void) { return g_last_error; }

int far_version(void) { return FAR_VERSION; }

far_status far_create(far_ctx** ctx, int device) {
  if (ctx == nullptr) return FAR_ERR_INVALID_ARG;
  *ctx = nullptr;
  int n = 0;
  cudaError_t e = cudaGetDeviceCount(&n);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDeviceCount");
  if (device < 0 || device >= n) return FAR_ERR_INVALID_ARG;
  far_ctx* out = new (std::nothrow) far_ctx();
  if (out == nullptr) return FAR_ERR_INTERNAL;
  far_ctx& c = *out;
  c.device = device;
  if ((e = cudaDeviceGetAttribute(&c.sm_count, cudaDevAttrMultiProcessorCount, device)) != cudaSuccess ||
      (e = cudaDeviceGetAttribute(&c.cc_major, cudaDevAttrComputeCapabilityMajor, device)) != cudaSuccess ||
      (e = cudaDeviceGetAttribute(&c.cc_minor, cudaDevAttrComputeCapabilityMinor, device)) != cudaSuccess)
    { delete out; return cuda_fail(e, "cudaDeviceGetAttribute"); }
  if (c.cc_major != 10 || c.cc_minor != 0) {
    std::snprintf(g_last_error, sizeof(g_last_error),
                  "device %d has compute capability %d.%d; this library is built for sm_100a only",
                  device, c.cc_major, c.cc_minor);
    delete out;
    return FAR_ERR_UNSUPPORTED;
  }
  c.decode_max_rows = env_int("FAR_DECODE_MAX_ROWS", 80);
  c.decode_cluster = env_int("FAR_DECODE_CLUSTER", 0);  // 0: the measured rule
  c.prefill_threads = env_int("FAR_PREFILL_THREADS", 256);
  if (c.prefill_threads < 32) c.prefill_threads = 32;
  if (c.prefill_threads > far::kMaxThreads) c.prefill_threads = far::kMaxThreads;
  c.prefill_kernel = env_int("FAR_PREFILL_KERNEL", 1) != 0 ? 1 : 0;
  c.ring_ctas_per_sm = env_int("FAR_RING_CTAS_PER_SM", 0);  // 0: by segments per row
  if (c.ring_ctas_per_sm < 0) c.ring_ctas_per_sm = 0;
  if (c.ring_ctas_per_sm > 8) c.ring_ctas_per_sm = 8;
  c.ring_threads = env_int("FAR_RING_THREADS", 256);  // at most kRingMaxConsumers
  c.ring_threads_set = std::getenv("FAR_RING_THREADS") != nullptr;
  c.ring_slots_max = env_int("FAR_RING_SLOTS", 0);  // 0: by the 72 KiB rule
  c.tensor_reverse = env_int("FAR_TENSOR_REVERSE", 1) != 0;
  c.tensor_fused = env_int("FAR_TENSOR_FUSED", 1) != 0;
  c.ring_gamma_mode = env_int("FAR_RING_GAMMA_SMEM", -1);
  c.ring_wide = env_int("FAR_RING_WIDE", 1) != 0 ? 1 : 0;
  c.ring_wide2 = env_int("FAR_RING_WIDE2", 1) != 0 ? 1 : 0;
  c.ring_wide1 = env_int("FAR_RING_WIDE1", 1) != 0 ? 1 : 0;
  c.ring_wide_group = env_int("FAR_RING_WIDE_GROUP", 1) != 0 ? 1 : 0;
  if (c.ring_gamma_mode > 1) c.ring_gamma_mode = 1;
  if (c.ring_gamma_mode < -1) c.ring_gamma_mode = -1;
  if (c.ring_slots_max < 0) c.ring_slots_max = 0;
  if (c.ring_slots_max > 32) c.ring_slots_max = 32;
  if (c.ring_threads < 32) c.ring_threads = 32;
  if (c.ring_threads > far::kRingMaxConsumers) c.ring_threads = far::kRingMaxConsumers;
  c.pdl = env_int("FAR_PDL", 1) != 0 ? 1 : 0;
  c.ring_min_rows = env_int("FAR_RING_MIN_ROWS", 0);  // 0: the measured rule
  c.wait_limit_ns = 2000000000ull;
  c.stall_segment = -1;
  c.force_regime = FAR_REGIME_AUTO;
  if (const char* f = std::getenv("FAR_FORCE_REGIME")) {
    if (std::strcmp(f, "decode") == 0) c.force_regime = FAR_REGIME_DECODE;
    if (std::strcmp(f, "prefill") == 0) c.force_regime = FAR_REGIME_PREFILL;
  }

  int prev = -1;
  if ((e = cudaGetDevice(&prev)) != cudaSuccess) { delete out; return cuda_fail(e, "cudaGetDevice"); }
  if (prev != device && (e = cudaSetDevice(device)) != cudaSuccess) {
    delete out;
    return cuda_fail(e, "cudaSetDevice");
  }
  e = far::configure_kernels();
  if (prev != device) cudaSetDevice(prev);
  if (e != cudaSuccess) { delete out; return cuda_fail(e, "cudaFuncSetAttribute"); }
  *ctx = out;
  return FAR_OK;
}

far_status far_destroy(far_ctx* ctx) {
  if (ctx != nullptr) host_pipe_release(ctx);
  delete ctx;
  return FAR_OK;
}

far_status far_test_stall(far_ctx* ctx, int64_t segment, uint32_t wait_limit_us) {
  if (ctx == nullptr) return FAR_ERR_INVALID_ARG;
  ctx->stall_segment = segment < 0 ? -1 : segment;
  ctx->wait_limit_ns = wait_limit_us == 0 ? 2000000000ull : static_cast<uint64_t>(wait_limit_us) * 1000ull;
  return FAR_OK;
}

far_status far_set_regime(far_ctx* ctx, far_regime regime, int decode_max_rows) {
  if (ctx == nullptr) return FAR_ERR_INVALID_ARG;
  if (regime != FAR_REGIME_AUTO && regime != FAR_REGIME_DECODE && regime != FAR_REGIME_PREFILL)
    return FAR_ERR_INVALID_ARG;
  ctx->force_regime = regime;
  if (decode_max_rows >= 0) ctx->decode_max_rows = decode_max_rows;
  return FAR_OK;
}

far_status far_describe_launch(const far_ctx* ctx, int64_t rows, int64_t H, far_dtype dtype,
                               int W, int has_residual, int has_norm_out, far_launch_info* info) {
  return far_describe_launch_pattern(ctx, rows, H, dtype, W, has_residual, has_norm_out,
                                     FAR_AR_RESIDUAL_RMSNORM, info);
}

far_status far_describe_launch_pattern(const far_ctx* ctx, int64_t rows, int64_t H,
                                       far_dtype dtype, int W, int has_residual, int has_norm_out,
                                       far_pattern pattern, far_launch_info* info) {
  if (ctx == nullptr || info == nullptr || rows < 0) return FAR_ERR_INVALID_ARG;
  if (pattern < FAR_AR_RESIDUAL_RMSNORM || pattern > FAR_AR_RESIDUAL_RMSNORM_FP8_GROUP)
    return FAR_ERR_INVALID_ARG;
  if (W < 1 || W > FAR_MAX_W) return FAR_ERR_INVALID_ARG;
  if (dtype != FAR_BF16 && dtype != FAR_FP16) return FAR_ERR_INVALID_ARG;
  if (H <= 0 || H % far::kPackElems != 0 || H > far::kMaxH) return FAR_ERR_UNSUPPORTED;
  int prev = -1;
  cudaError_t e = cudaGetDevice(&prev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (prev != ctx->device && (e = cudaSetDevice(ctx->device)) != cudaSuccess)
    return cuda_fail(e, "cudaSetDevice");
  const far::Launch l =
      plan_call(ctx, rows, H, dtype, W + (has_residual ? 1 : 0), has_norm_out != 0, pattern);
  if (prev != ctx->device) cudaSetDevice(prev);
  info->regime = l.regime;
  info->ctas_per_row = l.cluster;
  info->rows_per_cta = l.rows_per_cta;
  info->threads_per_cta = l.threads;
  info->packs_per_thread = l.vpt;
  info->grid_ctas = l.grid;
  info->kernel = l.kernel;
  info->ring_slots = l.nslot;
  info->ring_gamma_smem = l.kernel == 1 ? l.ring_gamma : 0;
  return FAR_OK;
}

far_status far_check(far_ctx* ctx, void* stream) {
  if (ctx == nullptr) return FAR_ERR_INVALID_ARG;
  int prev = -1;
  cudaError_t e = cudaGetDevice(&prev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (prev != ctx->device && (e = cudaSetDevice(ctx->device)) != cudaSuccess)
    return cuda_fail(e, "cudaSetDevice");
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned word = 0;
  e = far::read_error_word(&word, s);
  if (e == cudaSuccess && word != 0) e = far::clear_error_word(s);
  if (prev != ctx->device) cudaSetDevice(prev);
  if (e != cudaSuccess) return cuda_fail(e, "far_check");
  if (word != 0) {
    std::snprintf(g_last_error, sizeof(g_last_error),
                  "a bounded wait inside a kernel gave up (flags 0x%x); outputs of the "
                  "calls since the last far_check are not valid", word);
    return FAR_ERR_TIMEOUT;
  }
  return FAR_OK;
}

far_status far_validate(int64_t row_begin, int64_t row_end, const void* const* partials, int W,
                        const void* residual, const void* residual_out, const void* gamma,
                        int64_t T, int64_t H, far_dtype dtype, float eps, float weight_bias,
                        far_pattern pattern, const void* norm_out, const void* quant_out,
                        const float* scale_in, const float* scale_out) {
  if (W < 1 || W > FAR_MAX_W || partials == nullptr) return FAR_ERR_INVALID_ARG;
  if (T < 0 || H <= 0) return FAR_ERR_INVALID_ARG;
  if (dtype != FAR_BF16 && dtype != FAR_FP16) return FAR_ERR_INVALID_ARG;
  if (pattern != FAR_AR_RESIDUAL_RMSNORM && pattern != FAR_AR_RESIDUAL_RMSNORM_FP8_STATIC &&
      pattern != FAR_AR_RESIDUAL_RMSNORM_FP8_TOKEN && pattern != FAR_AR_RESIDUAL_RMSNORM_FP8_TENSOR &&
      pattern != FAR_AR_RESIDUAL_RMSNORM_FP8_GROUP)
    return FAR_ERR_INVALID_ARG;
  if (H % far::kPackElems != 0 || H > FAR_MAX_H) return FAR_ERR_UNSUPPORTED;
  if (row_begin < 0 || row_end < row_begin || row_end > T) return FAR_ERR_INVALID_ARG;
  if (T > INT64_MAX / (H * 2)) return FAR_ERR_INVALID_ARG;
  if (!std::isfinite(eps) || eps < 0.f || !std::isfinite(weight_bias)) return FAR_ERR_INVALID_ARG;
  if (T == 0) return FAR_OK;  // nothing is read or written: buffers are not checked
  if (gamma == nullptr) return FAR_ERR_INVALID_ARG;
  for (int r = 0; r < W; ++r)
    if (partials[r] == nullptr) return FAR_ERR_INVALID_ARG;
  if (pattern == FAR_AR_RESIDUAL_RMSNORM && norm_out == nullptr) return FAR_ERR_INVALID_ARG;
  if (pattern == FAR_AR_RESIDUAL_RMSNORM_FP8_STATIC && (quant_out == nullptr || scale_in == nullptr))
    return FAR_ERR_INVALID_ARG;
  if ((pattern == FAR_AR_RESIDUAL_RMSNORM_FP8_TOKEN || pattern == FAR_AR_RESIDUAL_RMSNORM_FP8_TENSOR ||
       pattern == FAR_AR_RESIDUAL_RMSNORM_FP8_GROUP) &&
      (quant_out == nullptr || scale_out == nullptr))
    return FAR_ERR_INVALID_ARG;

  // 16-byte packs everywhere; fp32 scales need 4 bytes.
  for (int r = 0; r < W; ++r)
    if (!aligned(partials[r], 16)) return FAR_ERR_ALIGNMENT;
  const void* tens[] = {residual, residual_out, gamma, norm_out, quant_out};
  for (const void* p : tens)
    if (p != nullptr && !aligned(p, 16)) return FAR_ERR_ALIGNMENT;
  if (scale_in != nullptr && !aligned(scale_in, 4)) return FAR_ERR_ALIGNMENT;
  if (scale_out != nullptr && !aligned(scale_out, 4)) return FAR_ERR_ALIGNMENT;

  // Outputs overlap no input and no other output.  The one exception is the
  // new residual written exactly over the residual (in place).
  {
    const int64_t tb = T * H * 2;
    const void* res_w = (residual_out != nullptr) ? residual_out : residual;  // may be null
    Range outs[4];
    int no = 0;
    if (res_w != nullptr) outs[no++] = span(res_w, tb);  // outs[0] when present
    if (norm_out != nullptr) outs[no++] = span(norm_out, tb);
    if (pattern != FAR_AR_RESIDUAL_RMSNORM) outs[no++] = span(quant_out, T * H);
    if (pattern == FAR_AR_RESIDUAL_RMSNORM_FP8_TOKEN || pattern == FAR_AR_RESIDUAL_RMSNORM_FP8_GROUP)
      outs[no++] = span(scale_out, T * 4);  // per group: the full extent is checked by far_fused_fp8_group
    if (pattern == FAR_AR_RESIDUAL_RMSNORM_FP8_TENSOR) outs[no++] = span(scale_out, 4);
    Range ins[FAR_MAX_W + 3];
    int ni = 0;
    for (int r = 0; r < W; ++r) ins[ni++] = span(partials[r], tb);
    const int res_in = (residual != nullptr) ? ni : -1;
    if (residual != nullptr) ins[ni++] = span(residual, tb);
    ins[ni++] = span(gamma, H * 2);
    if (pattern == FAR_AR_RESIDUAL_RMSNORM_FP8_STATIC) ins[ni++] = span(scale_in, 4);
    for (int i = 0; i < no; ++i) {
      for (int j = 0; j < ni; ++j) {
        if (!overlap(outs[i], ins[j])) continue;
        const bool in_place = (i == 0 && res_w != nullptr && j == res_in && res_w == residual);
        if (!in_place) return FAR_ERR_INVALID_ARG;
      }
      for (int j = i + 1; j < no; ++j)
        if (overlap(outs[i], outs[j])) return FAR_ERR_INVALID_ARG;
    }
  }
  return FAR_OK;
}

}  // extern "C"

namespace {

far::Params make_params(const void* const* partials, int W, const void* residual,
                        void* residual_out, const void* gamma, int64_t H, far_pattern pattern,
                        float eps, float weight_bias, void* norm_out, void* quant_out,
                        const float* scale_in, float* scale_out) {
  far::Params p{};
  for (int r = 0; r < W; ++r) p.partials[r] = partials[r];
  p.residual = residual;
  p.residual_out = (residual_out == nullptr) ? const_cast<void*>(residual) : residual_out;
  p.gamma = gamma;
  p.norm_out = norm_out;
  p.quant_out = (pattern == FAR_AR_RESIDUAL_RMSNORM) ? nullptr : static_cast<uint8_t*>(quant_out);
  p.scale_in = scale_in;
  p.scale_out = scale_out;
  p.W = W;
  p.H = static_cast<int>(H);
  p.packs = static_cast<int>(H / far::kPackElems);
  p.pattern = static_cast<int>(pattern);
  p.eps = eps;
  p.weight_bias = weight_bias;
  return p;
}

// Enqueue the kernels of rows [row_begin, row_end) with plan `whole`, in as
// many launches as the grid limits need (grid.y for decode clusters).
cudaError_t launch_rows(far::Params p, int dtype, const far::Launch& whole, int64_t row_begin,
                        int64_t row_end, cudaStream_t s) {
  const int64_t max_rows = whole.regime == FAR_REGIME_DECODE
                               ? 65535
                               : static_cast<int64_t>(0x7fffffff) * whole.rows_per_cta;
  cudaError_t e = cudaSuccess;
  for (int64_t b = row_begin; b < row_end && e == cudaSuccess; b += max_rows) {
    const int64_t n = (row_end - b < max_rows) ? (row_end - b) : max_rows;
    far::Launch l = whole;
    if (whole.regime == FAR_REGIME_DECODE)
      l.grid = n * l.cluster;
    else if (whole.kernel == 1)
      l.grid = (n < whole.grid) ? n : whole.grid;
    else
      l.grid = (n + l.rows_per_cta - 1) / l.rows_per_cta;
    p.row_begin = b;
    p.row_end = b + n;
    if (l.regime == FAR_REGIME_DECODE)
      e = far::launch_decode(p, dtype, l, s);
    else if (l.kernel == 1)
      e = far::launch_ring(p, dtype, l, s);
    else if (l.kernel == 2)
      e = far::launch_tensor_quant(p, dtype, l, s);
    else
      e = far::launch_prefill(p, dtype, l, s);
  }
  return e;
}

// Makes ctx's device current for the lifetime of the object.
struct DeviceGuard {
  int prev = -1;
  int dev;
  cudaError_t err = cudaSuccess;
  explicit DeviceGuard(int device) : dev(device) {
    err = cudaGetDevice(&prev);
    if (err == cudaSuccess && prev != dev) err = cudaSetDevice(dev);
  }
  ~DeviceGuard() {
    if (prev >= 0 && prev != dev) cudaSetDevice(prev);
  }
};

// The per-tensor path once its arguments are checked: zero the amax word,
// pass 1 (rinv of every row, the call's amax), pass 2 (the outputs).  The
// workspace holds the amax word at byte 0 and rinv[rows] from byte 256.
//
// Without norm_out, and with a new residual to write, pass 1 also stores
// each row's new residual (except in rows that may overflow the format,
// which it flags) and pass 2 forms the codes from it: the inputs are read
// once, and pass 2 moves 3 bytes per element.  When pass 1 is the ring
// kernel, pass 2 runs inside the same launch after a grid barrier.  With norm_out, whose
// 2-byte result would feel the rounding of y, or with no residual output,
// pass 2 reads every input again and writes every output, as pass 1's
// kernel would.
far_status far_fused_fp8_tensor_launch(far_ctx* ctx, int64_t row_begin, int64_t row_end,
                                       const void* const* partials, int W, const void* residual,
                                       void* residual_out, const void* gamma, int64_t H,
                                       far_dtype dtype, float eps, float weight_bias,
                                       void* norm_out, void* quant_out, float* scale_out,
                                       void* workspace, void* stream) {
  far::Params p = make_params(partials, W, residual, residual_out, gamma, H,
                              FAR_AR_RESIDUAL_RMSNORM_FP8_TENSOR, eps, weight_bias, norm_out,
                              quant_out, nullptr, scale_out);
  p.wait_limit_ns = ctx->wait_limit_ns;
  p.stall_segment = ctx->stall_segment;
  p.ws_amax = static_cast<unsigned*>(workspace);
  p.ws_done = p.ws_amax + 1;
  p.ws_claim = p.ws_amax + 2;
  p.ws_claim2 = p.ws_amax + 3;
  // second-pass rows per claim: about 1024 packs (16 KiB of each stored
  // row) per claim, so that a claim's rows outlast the next claim's round
  // trip, and the rows left over when the counter runs dry stay few
  {
    const int64_t packs = H / far::kPackElems;
    p.tail_chunk = static_cast<int>(packs >= 1024 ? 1 : (1024 / packs > 8 ? 8 : 1024 / packs));
  }
  p.ws_rinv = reinterpret_cast<float*>(static_cast<unsigned char*>(workspace) + 256);
  p.ws_row0 = row_begin;
  // what the second pass forms the codes from: norm_out when the call
  // writes it (the first pass stores it), else the new residual when there
  // is one to store, else the inputs read again
  p.tensor_source = norm_out != nullptr ? 2 : (p.residual_out != nullptr ? 1 : 0);
  const bool from_stored = p.tensor_source != 0;
  DeviceGuard guard(ctx->device);
  if (guard.err != cudaSuccess) return cuda_fail(guard.err, "cudaSetDevice");
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const far::Launch whole = plan_call(ctx, row_end - row_begin, H, dtype,
                                      W + (residual != nullptr ? 1 : 0), norm_out != nullptr,
                                      FAR_AR_RESIDUAL_RMSNORM_FP8_TENSOR);
  // the amax word, the count of rows done and the two row counters start at
  // zero: a one-CTA kernel after the preceding work, so that the first pass
  // can still be launched with PDL (its set-up overlapping this kernel)
  cudaError_t e = far::launch_ws_zero(static_cast<unsigned*>(workspace), ctx->pdl, s);
  if (e != cudaSuccess) return cuda_fail(e, "kernel launch (per-tensor workspace)");
  far::Launch first = whole;
  first.pdl = ctx->pdl;
  p.pattern = far::kTensorAmax;
  // With the ring kernel and the codes formed from the stored new residual,
  // both passes run in one launch: the CTAs take first-pass rows from a
  // counter, wait until every row is done (a wait on rows, not on CTAs, so
  // no co-residency is needed), then write the codes, the rows taken last
  // first.
  const bool fused = ctx->tensor_fused && from_stored && first.regime == FAR_REGIME_PREFILL &&
                     first.kernel == 1 &&
                     row_end - row_begin <= 0x7fffffff;
  if (fused) p.tensor_fused = 1;
  e = launch_rows(p, dtype, first, row_begin, row_end, s);
  if (e != cudaSuccess) return cuda_fail(e, "kernel launch (per-tensor pass 1)");
  if (fused) return FAR_OK;
  p.tensor_fused = 0;
  // the second pass takes the rows last row first: the rows the first pass
  // wrote last are still in L2 when it starts
  p.pattern = far::kTensorQuant;
  p.reverse = ctx->tensor_reverse;
  far::Launch second = whole;
  if (from_stored) {
    // one CTA per row (or several short rows), loads straight into registers
    plan_prefill(static_cast<int>(H / far::kPackElems), far::kMaxThreads, &second);
    second.kernel = 2;
    second.grid = (row_end - row_begin + second.rows_per_cta - 1) / second.rows_per_cta;
    second.pdl = ctx->pdl;
  }
  e = launch_rows(p, dtype, second, row_begin, row_end, s);
  if (e != cudaSuccess) return cuda_fail(e, "kernel launch (per-tensor pass 2)");
  return FAR_OK;
}

bool group_size_ok(int g) { return g >= 8 && g <= 256 && (g & (g - 1)) == 0; }

// Per-group FP8, once far_validate passed: H must hold whole groups, and
// scale_out (T x H / group_size floats) may overlap no other buffer.
far_status check_group_scales(const void* const* partials, int W, const void* residual,
                              const void* residual_out, const void* gamma, int64_t T, int64_t H,
                              int group_size, const void* norm_out, const void* quant_out,
                              const float* scale_out) {
  if (H % group_size != 0) return FAR_ERR_UNSUPPORTED;
  if (T > 0) {
    const Range sc = span(scale_out, T * (H / group_size) * 4);
    const int64_t tb = T * H * 2;
    for (int r = 0; r < W; ++r)
      if (overlap(sc, span(partials[r], tb))) return FAR_ERR_INVALID_ARG;
    const void* bufs16[] = {residual, residual_out, norm_out};
    for (const void* b : bufs16)
      if (b != nullptr && overlap(sc, span(b, tb))) return FAR_ERR_INVALID_ARG;
    if (overlap(sc, span(gamma, H * 2)) || overlap(sc, span(quant_out, T * H)))
      return FAR_ERR_INVALID_ARG;
  }
  return FAR_OK;
}

// ---------------------------------------------------------------------------
// far_fused_host: host buffers through a device staging area, in chunks of
// rows.  Chunk c uses staging buffer c % 2; its copy in (stream host_h2d),
// its kernel (the caller's stream) and its copy out (stream host_d2h) are
// ordered by events, so chunk c+1 is copied in and chunk c-1 copied out
// while chunk c runs.
// ---------------------------------------------------------------------------

size_t round256(int64_t x) { return static_cast<size_t>((x + 255) / 256 * 256); }

// About 64 MiB of inputs per chunk: measured on B200 over PCIe with the
// W=4 8192 x 8192 workload, 4 / 8 / 16 / 32 / 64 MiB chunks gave 47 / 54 /
// 60 / 64 / 65 GB/s end to end (fewer, larger copies; the first chunk's
// copy in and the last one's copy out are the only parts not overlapped).
int64_t default_chunk_rows(int W, int64_t H) {
  const int64_t row_in = static_cast<int64_t>(W + 1) * H * 2;  // bytes copied in per row
  const int64_t r = (int64_t{64} << 20) / row_in;
  return r > 0 ? r : 1;
}

// Staging layout: [gamma | scale_in | buffer 0 | buffer 1], every part
// 256-byte aligned; a buffer is [W partials | residual | residual_out |
// norm_out | quant_out | scale_out] for `rows` rows, with room for the
// largest scale_out (one per group of 8 elements).
struct Staging {
  size_t seg;      // one (rows, H) block of 2-byte elements
  size_t codes;    // the (rows, H) block of FP8 codes
  size_t scales;   // rows * H / 8 floats
  size_t head;     // gamma, then scale_in
  size_t per_buf;
  size_t total;
};

Staging staging_layout(int W, int64_t H, int64_t rows) {
  Staging L;
  L.seg = round256(rows * H * 2);
  L.codes = round256(rows * H);
  L.scales = round256(rows * (H / 8) * 4);
  L.head = round256(H * 2) + 256;
  L.per_buf = static_cast<size_t>(W + 3) * L.seg + L.codes + L.scales;
  L.total = L.head + 2 * L.per_buf;
  return L;
}

far_status host_pipe_ready(far_ctx* ctx) {
  if (ctx->host_ready) return FAR_OK;
  cudaError_t e = cudaSuccess;
  cudaStream_t s[2] = {nullptr, nullptr};
  cudaEvent_t ev[7] = {};
  for (int i = 0; i < 2 && e == cudaSuccess; ++i) e = cudaStreamCreateWithFlags(&s[i], cudaStreamNonBlocking);
  for (int i = 0; i < 7 && e == cudaSuccess; ++i) e = cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming);
  if (e != cudaSuccess) {
    for (cudaStream_t x : s)
      if (x != nullptr) cudaStreamDestroy(x);
    for (cudaEvent_t x : ev)
      if (x != nullptr) cudaEventDestroy(x);
    return cuda_fail(e, "far_fused_host: creating its streams and events");
  }
  ctx->host_h2d = s[0];
  ctx->host_d2h = s[1];
  ctx->host_start = ev[0];
  for (int b = 0; b < 2; ++b) {
    ctx->host_in[b] = ev[1 + b];
    ctx->host_comp[b] = ev[3 + b];
    ctx->host_out[b] = ev[5 + b];
  }
  ctx->host_ready = true;
  return FAR_OK;
}

}  // namespace

extern "C" {

far_status far_fused_rows(far_ctx* ctx, int64_t row_begin, int64_t row_end,
                          const void* const* partials, int W, const void* residual,
                          void* residual_out, const void* gamma, int64_t T, int64_t H,
                          far_dtype dtype, float eps, float weight_bias, far_pattern pattern,
                          void* norm_out, void* quant_out, const float* scale_in, float* scale_out,
                          void* stream) {
  if (ctx == nullptr) return FAR_ERR_INVALID_ARG;
  // the per-tensor pattern needs a workspace (far_fused_fp8_tensor), the
  // per-group one a group size (far_fused_fp8_group)
  if (pattern == FAR_AR_RESIDUAL_RMSNORM_FP8_TENSOR || pattern == FAR_AR_RESIDUAL_RMSNORM_FP8_GROUP)
    return FAR_ERR_INVALID_ARG;
  far_status st = far_validate(row_begin, row_end, partials, W, residual, residual_out, gamma, T, H,
                               dtype, eps, weight_bias, pattern, norm_out, quant_out, scale_in,
                               scale_out);
  if (st != FAR_OK) return st;
  if (row_end == row_begin) return FAR_OK;

  far::Params p = make_params(partials, W, residual, residual_out, gamma, H, pattern, eps,
                              weight_bias, norm_out, quant_out, scale_in, scale_out);
  p.wait_limit_ns = ctx->wait_limit_ns;
  p.stall_segment = ctx->stall_segment;
  DeviceGuard guard(ctx->device);
  if (guard.err != cudaSuccess) return cuda_fail(guard.err, "cudaSetDevice");
  const far::Launch whole = plan(ctx, row_end - row_begin, H, dtype, W + (residual != nullptr ? 1 : 0),
                   norm_out != nullptr);
  const cudaError_t e = launch_rows(p, dtype, whole, row_begin, row_end, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
  return FAR_OK;
}

size_t far_fp8_tensor_workspace_bytes(int64_t rows) {
  if (rows < 0) rows = 0;
  return static_cast<size_t>((256 + 4 * rows + 255) / 256 * 256);
}

far_status far_fused_fp8_tensor(far_ctx* ctx, int64_t row_begin, int64_t row_end,
                                const void* const* partials, int W, const void* residual,
                                void* residual_out, const void* gamma, int64_t T, int64_t H,
                                far_dtype dtype, float eps, float weight_bias, void* norm_out,
                                void* quant_out, float* scale_out, void* workspace,
                                size_t workspace_bytes, void* stream) {
  if (ctx == nullptr) return FAR_ERR_INVALID_ARG;
  far_status st = far_validate(row_begin, row_end, partials, W, residual, residual_out, gamma, T, H,
                               dtype, eps, weight_bias, FAR_AR_RESIDUAL_RMSNORM_FP8_TENSOR, norm_out,
                               quant_out, nullptr, scale_out);
  if (st != FAR_OK) return st;
  if (row_end == row_begin) return FAR_OK;
  const int64_t rows = row_end - row_begin;
  if (workspace == nullptr || workspace_bytes < far_fp8_tensor_workspace_bytes(rows))
    return FAR_ERR_INVALID_ARG;
  if (!aligned(workspace, 256)) return FAR_ERR_ALIGNMENT;
  // the workspace is written: it may overlap no argument buffer
  {
    const Range ws = span(workspace, static_cast<int64_t>(far_fp8_tensor_workspace_bytes(rows)));
    const int64_t tb = T * H * 2;
    for (int r = 0; r < W; ++r)
      if (overlap(ws, span(partials[r], tb))) return FAR_ERR_INVALID_ARG;
    const void* bufs16[] = {residual, residual_out, norm_out};
    for (const void* b : bufs16)
      if (b != nullptr && overlap(ws, span(b, tb))) return FAR_ERR_INVALID_ARG;
    if (overlap(ws, span(gamma, H * 2)) || overlap(ws, span(quant_out, T * H)) ||
        overlap(ws, span(scale_out, 4)))
      return FAR_ERR_INVALID_ARG;
  }
  return far_fused_fp8_tensor_launch(ctx, row_begin, row_end, partials, W, residual, residual_out,
                                     gamma, H, dtype, eps, weight_bias, norm_out, quant_out,
                                     scale_out, workspace, stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Per-tensor FP8 with the library's own scratch instead of a workspace
// ---------------------------------------------------------------------------

namespace {

// The scratch of far_fused_fp8_tensor_noalloc: the amax word at byte 0 and
// one rinv per row from byte 256, for at most FAR_FP8_TENSOR_NOALLOC_MAX_ROWS
// rows (256 KiB + 256 bytes).  It is part of the library image: every GPU
// that loads the library holds it until the process exits, and every call
// on that GPU shares it.
static __device__ __align__(256) unsigned char g_noalloc_scratch[256 + 4 * FAR_FP8_TENSOR_NOALLOC_MAX_ROWS];

// Device address of g_noalloc_scratch for each device ordinal, looked up
// on the first call on that device.  In host code the array's name only
// stands for the symbol, so the kernels get this address instead.
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[256] = {};

}  // namespace

extern "C" {

far_status far_fused_fp8_tensor_noalloc(far_ctx* ctx, int64_t row_begin, int64_t row_end,
                                        const void* const* partials, int W, const void* residual,
                                        void* residual_out, const void* gamma, int64_t T,
                                        int64_t H, far_dtype dtype, float eps, float weight_bias,
                                        void* norm_out, void* quant_out, float* scale_out,
                                        void* stream) {
  if (ctx == nullptr) return FAR_ERR_INVALID_ARG;
  far_status st = far_validate(row_begin, row_end, partials, W, residual, residual_out, gamma, T, H,
                               dtype, eps, weight_bias, FAR_AR_RESIDUAL_RMSNORM_FP8_TENSOR, norm_out,
                               quant_out, nullptr, scale_out);
  if (st != FAR_OK) return st;
  if (row_end - row_begin > FAR_FP8_TENSOR_NOALLOC_MAX_ROWS) {
    std::snprintf(g_last_error, sizeof(g_last_error),
                  "far_fused_fp8_tensor_noalloc handles at most %d rows per call (got %lld); "
                  "use far_fused_fp8_tensor with a workspace",
                  FAR_FP8_TENSOR_NOALLOC_MAX_ROWS, static_cast<long long>(row_end - row_begin));
    return FAR_ERR_UNSUPPORTED;
  }
  if (row_end == row_begin) return FAR_OK;
  if (ctx->device < 0 || ctx->device >= 256) {
    std::snprintf(g_last_error, sizeof(g_last_error),
                  "far_fused_fp8_tensor_noalloc keeps its scratch address for device "
                  "ordinals 0-255 only (device %d)", ctx->device);
    return FAR_ERR_UNSUPPORTED;
  }

  void* scratch = nullptr;
  {
    DeviceGuard guard(ctx->device);  // the lookup needs the device current
    if (guard.err != cudaSuccess) return cuda_fail(guard.err, "cudaSetDevice");
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (g_noalloc_ptr[ctx->device] == nullptr) {
      void* ptr = nullptr;
      const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
      if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress");
      g_noalloc_ptr[ctx->device] = ptr;
    }
    scratch = g_noalloc_ptr[ctx->device];
  }
  // the same two passes as far_fused_fp8_tensor, which zero the amax word first
  return far_fused_fp8_tensor_launch(ctx, row_begin, row_end, partials, W, residual, residual_out,
                                     gamma, H, dtype, eps, weight_bias, norm_out, quant_out,
                                     scale_out, scratch, stream);
}

far_status far_fused_fp8_group(far_ctx* ctx, int64_t row_begin, int64_t row_end,
                               const void* const* partials, int W, const void* residual,
                               void* residual_out, const void* gamma, int64_t T, int64_t H,
                               far_dtype dtype, float eps, float weight_bias, int group_size,
                               void* norm_out, void* quant_out, float* scale_out, void* stream) {
  if (ctx == nullptr) return FAR_ERR_INVALID_ARG;
  if (!group_size_ok(group_size)) return FAR_ERR_UNSUPPORTED;
  far_status st = far_validate(row_begin, row_end, partials, W, residual, residual_out, gamma, T, H,
                               dtype, eps, weight_bias, FAR_AR_RESIDUAL_RMSNORM_FP8_GROUP, norm_out,
                               quant_out, nullptr, scale_out);
  if (st != FAR_OK) return st;
  st = check_group_scales(partials, W, residual, residual_out, gamma, T, H, group_size, norm_out,
                          quant_out, scale_out);
  if (st != FAR_OK) return st;
  if (row_end == row_begin) return FAR_OK;

  far::Params p = make_params(partials, W, residual, residual_out, gamma, H,
                              FAR_AR_RESIDUAL_RMSNORM_FP8_GROUP, eps, weight_bias, norm_out,
                              quant_out, nullptr, scale_out);
  p.wait_limit_ns = ctx->wait_limit_ns;
  p.stall_segment = ctx->stall_segment;
  p.group_lanes = group_size / far::kPackElems;
  p.groups_per_row = static_cast<int>(H / group_size);
  DeviceGuard guard(ctx->device);
  if (guard.err != cudaSuccess) return cuda_fail(guard.err, "cudaSetDevice");
  const far::Launch whole = plan_call(ctx, row_end - row_begin, H, dtype,
                                      W + (residual != nullptr ? 1 : 0), norm_out != nullptr,
                                      FAR_AR_RESIDUAL_RMSNORM_FP8_GROUP);
  const cudaError_t e = launch_rows(p, dtype, whole, row_begin, row_end, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
  return FAR_OK;
}

far_status far_fused(far_ctx* ctx, const void* const* partials, int W, const void* residual,
                     void* residual_out, const void* gamma, int64_t T, int64_t H, far_dtype dtype,
                     float eps, float weight_bias, far_pattern pattern, void* norm_out,
                     void* quant_out, const float* scale_in, float* scale_out, void* stream) {
  return far_fused_rows(ctx, 0, T, partials, W, residual, residual_out, gamma, T, H, dtype, eps,
                        weight_bias, pattern, norm_out, quant_out, scale_in, scale_out, stream);
}

size_t far_host_staging_bytes(int W, int64_t H, int64_t chunk_rows) {
  if (W < 1 || W > FAR_MAX_W || H <= 0 || H % far::kPackElems != 0 || H > far::kMaxH) return 0;
  const int64_t rows = chunk_rows > 0 ? chunk_rows : default_chunk_rows(W, H);
  return staging_layout(W, H, rows).total;
}

far_status far_fused_host(far_ctx* ctx, const void* const* partials, int W, const void* residual,
                          void* residual_out, const void* gamma, int64_t T, int64_t H,
                          far_dtype dtype, float eps, float weight_bias, far_pattern pattern,
                          int group_size, void* norm_out, void* quant_out, const float* scale_in,
                          float* scale_out, int64_t chunk_rows, void* staging,
                          size_t staging_bytes, void* stream) {
  if (ctx == nullptr) return FAR_ERR_INVALID_ARG;
  if (pattern == FAR_AR_RESIDUAL_RMSNORM_FP8_TENSOR) {
    std::snprintf(g_last_error, sizeof(g_last_error),
                  "far_fused_host: per-tensor FP8 needs every row before any code; "
                  "use far_fused_fp8_tensor on device buffers");
    return FAR_ERR_UNSUPPORTED;
  }
  const bool group = pattern == FAR_AR_RESIDUAL_RMSNORM_FP8_GROUP;
  if (group && !group_size_ok(group_size)) return FAR_ERR_UNSUPPORTED;
  far_status st = far_validate(0, T, partials, W, residual, residual_out, gamma, T, H, dtype, eps,
                               weight_bias, pattern, norm_out, quant_out, scale_in, scale_out);
  if (st != FAR_OK) return st;
  if (group) {
    st = check_group_scales(partials, W, residual, residual_out, gamma, T, H, group_size,
                            norm_out, quant_out, scale_out);
    if (st != FAR_OK) return st;
  }
  if (chunk_rows < 0) return FAR_ERR_INVALID_ARG;
  if (T == 0) return FAR_OK;
  int64_t R = chunk_rows > 0 ? chunk_rows : default_chunk_rows(W, H);
  const Staging L = staging_layout(W, H, R);  // sized for R rows, as the caller's query
  if (R > T) R = T;
  if (staging == nullptr || staging_bytes < L.total) return FAR_ERR_INVALID_ARG;
  if (!aligned(staging, 256)) return FAR_ERR_ALIGNMENT;

  DeviceGuard guard(ctx->device);
  if (guard.err != cudaSuccess) return cuda_fail(guard.err, "cudaSetDevice");
  std::lock_guard<std::mutex> lock(ctx->host_mu);
  st = host_pipe_ready(ctx);
  if (st != FAR_OK) return st;

  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const cudaStream_t in = ctx->host_h2d, out = ctx->host_d2h;
  unsigned char* const base = static_cast<unsigned char*>(staging);
  const int64_t rb = H * 2;  // bytes of one row of 2-byte elements
  // where the new residual goes: residual_out, else in place into residual
  void* const h_rout = residual_out != nullptr ? residual_out : const_cast<void*>(residual);
  const int64_t nsc = pattern == FAR_AR_RESIDUAL_RMSNORM_FP8_TOKEN ? 1
                      : group                                      ? H / group_size
                                                                   : 0;  // scales per row
  cudaError_t e = cudaSuccess;
#define FAR_HOST_CK(call, what)                 \
  do {                                          \
    if ((e = (call)) != cudaSuccess) return cuda_fail(e, "far_fused_host: " what); \
  } while (0)

  // copies start after the caller's earlier work on `stream`, and the head
  // (gamma, scale_in) is rewritten only after the kernels of the previous
  // call on this context, which read it, are done (an event never recorded
  // makes no one wait)
  FAR_HOST_CK(cudaEventRecord(ctx->host_start, s), "cudaEventRecord");
  FAR_HOST_CK(cudaStreamWaitEvent(in, ctx->host_start, 0), "cudaStreamWaitEvent");
  FAR_HOST_CK(cudaStreamWaitEvent(in, ctx->host_comp[0], 0), "cudaStreamWaitEvent");
  FAR_HOST_CK(cudaStreamWaitEvent(in, ctx->host_comp[1], 0), "cudaStreamWaitEvent");
  // gamma and the static scale, once per call
  FAR_HOST_CK(cudaMemcpyAsync(base, gamma, static_cast<size_t>(rb), cudaMemcpyHostToDevice, in),
              "copy of gamma");
  float* const d_scale_in = reinterpret_cast<float*>(base + round256(rb));
  if (pattern == FAR_AR_RESIDUAL_RMSNORM_FP8_STATIC)
    FAR_HOST_CK(cudaMemcpyAsync(d_scale_in, scale_in, 4, cudaMemcpyHostToDevice, in),
                "copy of scale_in");

  const int64_t nchunks = (T + R - 1) / R;
  for (int64_t c = 0; c < nchunks; ++c) {
    const int b = static_cast<int>(c & 1);
    const int64_t r0 = c * R;
    const int64_t n = T - r0 < R ? T - r0 : R;
    unsigned char* const buf = base + L.head + b * L.per_buf;
    unsigned char* const d_res = buf + W * L.seg;
    unsigned char* const d_rout = d_res + L.seg;
    unsigned char* const d_norm = d_rout + L.seg;
    unsigned char* const d_quant = d_norm + L.seg;
    float* const d_scale = reinterpret_cast<float*>(d_quant + L.codes);

    // copy in, once buffer b's previous chunk (in this call or an earlier
    // one on this context) has been copied out; an event never recorded
    // makes no one wait
    FAR_HOST_CK(cudaStreamWaitEvent(in, ctx->host_out[b], 0), "cudaStreamWaitEvent");
    const void* d_parts[far::kMaxW];
    for (int r = 0; r < W; ++r) {
      d_parts[r] = buf + r * L.seg;
      FAR_HOST_CK(cudaMemcpyAsync(buf + r * L.seg, static_cast<const unsigned char*>(partials[r]) + r0 * rb,
                                  static_cast<size_t>(n * rb), cudaMemcpyHostToDevice, in),
                  "copy in of a partial");
    }
    if (residual != nullptr)
      FAR_HOST_CK(cudaMemcpyAsync(d_res, static_cast<const unsigned char*>(residual) + r0 * rb,
                                  static_cast<size_t>(n * rb), cudaMemcpyHostToDevice, in),
                  "copy in of the residual");
    FAR_HOST_CK(cudaEventRecord(ctx->host_in[b], in), "cudaEventRecord");

    // the kernel, on the caller's stream (no programmatic launch: it follows
    // an event wait, not a kernel)
    FAR_HOST_CK(cudaStreamWaitEvent(s, ctx->host_in[b], 0), "cudaStreamWaitEvent");
    far::Params p = make_params(d_parts, W, residual != nullptr ? d_res : nullptr,
                                h_rout != nullptr ? d_rout : nullptr, base, H, pattern, eps,
                                weight_bias, norm_out != nullptr ? d_norm : nullptr,
                                quant_out != nullptr ? d_quant : nullptr,
                                pattern == FAR_AR_RESIDUAL_RMSNORM_FP8_STATIC ? d_scale_in : nullptr,
                                nsc > 0 ? d_scale : nullptr);
    p.wait_limit_ns = ctx->wait_limit_ns;
    p.stall_segment = ctx->stall_segment;
    far::Launch l = plan_call(ctx, n, H, dtype, W + (residual != nullptr ? 1 : 0),
                              norm_out != nullptr, pattern);
    if (group) {
      p.group_lanes = group_size / far::kPackElems;
      p.groups_per_row = static_cast<int>(H / group_size);
    }
    l.pdl = 0;
    FAR_HOST_CK(launch_rows(p, dtype, l, 0, n, s), "kernel launch");
    FAR_HOST_CK(cudaEventRecord(ctx->host_comp[b], s), "cudaEventRecord");

    // copy out
    FAR_HOST_CK(cudaStreamWaitEvent(out, ctx->host_comp[b], 0), "cudaStreamWaitEvent");
    if (h_rout != nullptr)
      FAR_HOST_CK(cudaMemcpyAsync(static_cast<unsigned char*>(h_rout) + r0 * rb, d_rout,
                                  static_cast<size_t>(n * rb), cudaMemcpyDeviceToHost, out),
                  "copy out of residual_out");
    if (norm_out != nullptr)
      FAR_HOST_CK(cudaMemcpyAsync(static_cast<unsigned char*>(norm_out) + r0 * rb, d_norm,
                                  static_cast<size_t>(n * rb), cudaMemcpyDeviceToHost, out),
                  "copy out of norm_out");
    if (quant_out != nullptr)
      FAR_HOST_CK(cudaMemcpyAsync(static_cast<unsigned char*>(quant_out) + r0 * H, d_quant,
                                  static_cast<size_t>(n * H), cudaMemcpyDeviceToHost, out),
                  "copy out of quant_out");
    if (nsc > 0)
      FAR_HOST_CK(cudaMemcpyAsync(scale_out + r0 * nsc, d_scale, static_cast<size_t>(n * nsc * 4),
                                  cudaMemcpyDeviceToHost, out),
                  "copy out of scale_out");
    FAR_HOST_CK(cudaEventRecord(ctx->host_out[b], out), "cudaEventRecord");
  }
  // the caller's stream reaches the end of the call once every copy out is done
  FAR_HOST_CK(cudaStreamWaitEvent(s, ctx->host_out[0], 0), "cudaStreamWaitEvent");
  if (nchunks > 1) FAR_HOST_CK(cudaStreamWaitEvent(s, ctx->host_out[1], 0), "cudaStreamWaitEvent");
#undef FAR_HOST_CK
  return FAR_OK;
}

}  // extern "C"

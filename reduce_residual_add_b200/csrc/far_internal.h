// far_internal.h -- declarations shared by the ABI layer (far_abi.cu) and the
// kernels (far_kernels.cu).  Not installed; the public interface is far.h.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace far {

constexpr int kMaxW = 16;        // partial buffers per call
constexpr int kMaxH = 16384;     // longest row held in registers
constexpr int kPackElems = 8;    // 2-byte elements per 16-byte pack
constexpr int kMaxThreads = 256; // threads per row (CTA) in every kernel
constexpr int kRingSmemMax = 227 * 1024;  // dynamic shared memory of one ring CTA
constexpr int kRingMaxConsumers = 256;    // consumer threads of one ring CTA
constexpr int kRingWideConsumers = 384;   // ... of the wide build (4 packs per thread,
                                          // rows of 1025-1536 packs, 2 CTAs per SM)
constexpr int kRingWide2Consumers = 448;  // ... of the wide 2-pack build (rows of
                                          // 513-896 packs, 2 CTAs per SM)
constexpr int kRingWide1Consumers = 512;  // ... of the one-CTA wide build (4 packs
                                          // per thread, rows of 1537-2048 packs)

enum Dtype : int { kBf16 = 0, kFp16 = 1 };
enum Pattern : int {
  kNormOnly = 0,
  kFp8Static = 1,
  kFp8Token = 2,
  kFp8Tensor = 3,       // public value of dynamic per-tensor FP8
  kFp8Group = 4,        // per-group FP8: one scale per group of consecutive elements
  kTensorAmax = 16,     // its first pass: rinv of each row + the call's amax
  kTensorQuant = 17     // its second pass: the other outputs, from the stored rinv and amax
};

// Everything one launch needs, passed by value in the kernel's parameter
// space (about 200 bytes).
struct Params {
  const void* partials[kMaxW];  // W read-only (T, H) tensors
  const void* residual;         // (T, H) or null
  void* residual_out;           // (T, H) or null (may equal residual)
  const void* gamma;            // (H,)
  void* norm_out;               // (T, H) or null
  uint8_t* quant_out;           // (T, H) e4m3 codes or null
  const float* scale_in;        // static FP8 scale (1 float) or null
  float* scale_out;             // per-row FP8 scales (T floats) or null
  int64_t row_begin;            // rows [row_begin, row_end) of the T-row tensors
  int64_t row_end;
  int W;
  int H;
  int packs;                    // H / 8
  int pattern;
  float eps;
  float weight_bias;
  float* ws_rinv;               // per-tensor FP8: rinv of row t at ws_rinv[t - ws_row0]
  unsigned* ws_amax;            // per-tensor FP8: the call's amax as fp32 bits
  int64_t ws_row0;              // per-tensor FP8: first row of the call
  int group_lanes;              // per-group FP8: 16-byte packs per group (power of two <= 32)
  int groups_per_row;           // per-group FP8: H / group size
  uint64_t wait_limit_ns;       // every bounded wait gives up after this long
  int64_t stall_segment;        // test hook: the ring producer skips this copy (-1: none)
  int reverse;                  // take the rows from row_end - 1 down to row_begin
  int tensor_source;            // per-tensor FP8: what the second pass forms the codes
                                // from -- 0 the inputs again, 1 the new residual the
                                // first pass stores, 2 the norm_out it stores
  int tensor_fused;             // per-tensor FP8 in one ring launch: the CTAs take rows
                                // from a shared counter (ws_claim), wait until every
                                // row is done (ws_done), then write the codes from the
                                // stored new residual or norm_out, the last quarter
                                // of rows in chunks from a second counter (ws_claim2)
  unsigned* ws_done;            // per-tensor FP8, one launch: rows past the first pass
  unsigned* ws_claim;           // per-tensor FP8, one launch: rows taken so far
  unsigned* ws_claim2;          // ... second-pass rows taken so far
  int tail_chunk;               // ... second-pass rows taken per claim (1-32)
};

// Geometry of one launch, chosen on the host.
struct Launch {
  int regime;           // 1 decode (cluster per row), 2 prefill
  int kernel;           // prefill: 0 direct loads, 1 TMA bulk-copy ring,
                        // 2 per-tensor FP8 second pass from the stored new residual
  int cluster;          // CTAs per row (decode)
  int vpt;              // 16-byte packs per thread
  int tpr;              // threads per row (prefill) / per CTA (decode)
  int rows_per_cta;     // prefill
  int threads;          // threads per CTA
  int64_t grid;         // CTAs
  int nslot;            // ring: shared-memory slots of one row segment each
  int smem_bytes;       // ring: dynamic shared memory per CTA
  int pdl;              // launch with programmatic stream serialization
  int ring_minb;        // ring: CTAs per SM its registers are sized for (2 or 3; 1 or 2 at 8 packs)
  int ring_gamma;       // ring: 1 = gamma staged in shared memory, 0 = read through L1
  int ring_wide;        // ring: the wide build (up to kRingWideConsumers consumers)
};

// Enqueue one kernel on `stream`.  Returns the launch error (cudaSuccess if
// the launch was accepted).
cudaError_t launch_prefill(const Params& p, int dtype, const Launch& l, cudaStream_t stream);
cudaError_t launch_decode(const Params& p, int dtype, const Launch& l, cudaStream_t stream);
cudaError_t launch_ring(const Params& p, int dtype, const Launch& l, cudaStream_t stream);
cudaError_t launch_tensor_quant(const Params& p, int dtype, const Launch& l, cudaStream_t stream);
// Zero the per-tensor workspace's first four words, after the preceding
// kernels in the stream (a kernel, so that the next launch may use PDL).
cudaError_t launch_ws_zero(unsigned* ws, int pdl, cudaStream_t stream);

// Bytes of the ring kernel's shared memory before its first slot.
int ring_header_bytes(int nslot);

// Resident ring CTAs per SM for this configuration on the current device
// (0 if it cannot run).
int ring_occupancy(int dtype, int vpt, int minb, int threads, int smem_bytes);

// Resident decode-kernel CTAs per SM at `threads` threads (its clusters
// aside; 0 if it cannot run).
int decode_occupancy(int dtype, int vpt, int threads);

// The device error word of the current device (see far_check): read it
// after the work on `stream`, or clear it.  Both synchronise `stream`.
cudaError_t read_error_word(unsigned* out, cudaStream_t stream);
cudaError_t clear_error_word(cudaStream_t stream);

// One-time per-device set-up of kernel attributes (non-portable cluster
// sizes).  Call with the device current.
cudaError_t configure_kernels();

}  // namespace far

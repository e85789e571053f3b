// Internal declarations shared by libkda's translation units (not installed).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kda.h"

namespace kda {

constexpr int kChunk = 64;   // tokens per chunk of the prefill

// How the decay is given: one log_alpha per key channel (KDA), one per token and
// head (Gated DeltaNet), or none (DeltaNet, alpha = 1).
enum GateKind { KDA_GATE_NONE = 0, KDA_GATE_SCALAR = 1, KDA_GATE_CHANNEL = 2 };

struct ForwardArgs {
    const void *q, *k, *v;
    const float *log_alpha, *beta;
    const float *s0;          // may be null (zero state)
    float *out;
    float *sT;                // may be null
    int B, T, H, dk, dv;
    kda_dtype dtype;
    float scale;
    int gate;                 // GateKind
    int prep_flags;           // kPrep* (two-kernel prefill only)
};

// Optional steps before the path, fused into the two-kernel prefill's first kernel:
// log_alpha holds gate pre-activations x and log alpha = log(sigmoid(x)); q and k
// rows are L2-normalised (a zero row stays zero).
constexpr int kPrepLogsigmoidGate = 1, kPrepNormalizeQK = 2;

struct DecodeArgs {
    const void *q, *k, *v;
    const float *log_alpha, *beta;
    float *state;
    float *out;
    int B, H, dk, dv;
    kda_dtype dtype;
    float scale;
    int gate;                 // GateKind
};

// Each launcher enqueues its kernel(s) on `stream` and returns the launch
// status.  Arguments are already validated by the C-ABI layer.
cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t stream);
cudaError_t launch_prefill_simt(const ForwardArgs &a, cudaStream_t stream);
// Tensor-core (tcgen05) prefill: bf16 inputs with dk = dv = 128.
bool prefill_tc_supported(const ForwardArgs &a);
cudaError_t launch_prefill_tc(const ForwardArgs &a, cudaStream_t stream);
// Tensor-core prefill with one decay per token and head (or none): bf16, dk = dv = 128.
cudaError_t launch_prefill_gdn_tc(const ForwardArgs &a, cudaStream_t stream);
cudaError_t take_gdn_device_status(unsigned int *status);
// Two-kernel tensor-core prefill (chunk-local kernel, then the state chain) with a
// caller-provided workspace: bf16, dk = dv = 128, per-channel gate.
bool prefill_split_supported(const ForwardArgs &a);
size_t prefill_split_workspace_full(int B, int T, int H);   // whole sequence in one block
size_t prefill_split_workspace_best(int B, int T, int H);   // the fastest schedule's workspace
size_t prefill_split_workspace_min(int B, int T, int H);    // one chunk per block + state carry
// The chain runs one CTA per (b, h) when the heads fill the SMs, or when the sequence
// is long and the heads few enough that the chunk-local kernel of the next block runs
// beside it (pipelined over two workspace slots), else one CTA per (b, h, 32-column
// slice).  T_whole: the length of the whole sequence when a is one block of it (the
// host-memory path), so that the kernel choice is the whole sequence's.
bool split_per_head(int B, int T_whole, int H);
cudaError_t launch_prefill_split(const ForwardArgs &a, uint8_t *ws, size_t ws_bytes, cudaStream_t stream,
                                 int T_whole = 0);
cudaError_t take_split_device_status(unsigned int *status);
// Time-axis split (the chain is linear in (U, S_0)), one contiguous segment of the
// sequence per call; the workspace holds the whole segment's records:
//   local:   outputs and final state (a.sT) from a.s0 (zero if null), and the
//            transfer [B,H,dk,dk] = the state alone propagated from I;
//   correct: out += outputs of `start` propagated alone; a.sT = local_final + that state;
//   compose: start = F_0, then F_j + P_j start for j = 1..R-1 (fp32).
cudaError_t launch_segment_local(const ForwardArgs &a, float *transfer, uint8_t *ws, cudaStream_t stream);
cudaError_t launch_segment_correct(const ForwardArgs &a, const float *start, const float *local_final,
                                   const uint8_t *ws, cudaStream_t stream);
cudaError_t launch_affine_compose(const float *transfers, const float *local_finals, int R, int BH, float *start,
                                  cudaStream_t stream);
// Backward pass (fp32 CUDA cores; bf16 or fp32 inputs; dk = dv = D in {64, 128}).
// The workspace holds the forward state before every 8th token and the adjoint at
// the end of every chunk: backward_workspace_bytes(B, T, H, D) bytes.
struct BackwardArgs {
    const void *q, *k, *v;
    const float *log_alpha, *beta;
    const float *s0;          // may be null (zero initial state)
    const float *d_out;
    const float *d_final;     // may be null (no cotangent of the final state)
    float *dq, *dk, *dv, *dlog_alpha, *dbeta;
    float *d_s0;              // may be null
    int B, T, H, Dk, Dv;      // head dims (equal)
    kda_dtype dtype;
    float scale;
    void *workspace;
};
size_t backward_workspace_bytes(int B, int T, int H, int D);
cudaError_t launch_backward(const BackwardArgs &a, cudaStream_t stream);
// One CTA whose bounded wait on a barrier nothing completes gives up after about
// wait_ms and records the device status bit (failure-path self-test).
cudaError_t launch_selftest_timeout(unsigned int wait_ms, cudaStream_t stream);
// Reads and clears the device status word the tensor-core kernels set when a
// bounded wait gives up (bit 0).  Synchronous.
cudaError_t take_device_status(unsigned int *status);

// Counts one kernel enqueued through the library (see kda_launch_count).
void note_launch();

// Loads of the two input dtypes as fp32 (bf16 -> fp32 is exact).
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

}  // namespace kda

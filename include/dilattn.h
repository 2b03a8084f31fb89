/*
 * dilattn -- LongNet dilated attention, forward and backward, on one B200
 * (sm_100a). C ABI: plain pointers and sizes, nothing from PyTorch.
 *
 * The operation (from the LongNet pages: the gptget.net summary of arXiv
 * 2307.02486, sections "方法论" and "方法详解"; its abstract, printed on every
 * page; and the DarcStar commentary on the darcstar.tech page):
 *
 *   For each pattern i = (w_i, r_i) and head h, the length-N sequence is cut
 *   into segments [s*w_i, min((s+1)*w_i, N)); segment s keeps rows
 *   s*w_i + (h mod r_i) + k*r_i below its end ("方法详解": equal segments,
 *   several dilation rates, a different offset per head). Softmax attention
 *   with scale 1/sqrt(d) runs on the kept rows of each segment, causal in
 *   position order when causal = 1 (abstract: a drop-in replacement for
 *   standard attention). The per-pattern results of a row are merged as
 *   O = sum_i Z_i O_i / sum_j Z_j, Z_i being pattern i's softmax
 *   denominator, carried as a log-sum-exp (DarcStar commentary: the shared
 *   denominator must stay exact). Rows no pattern keeps get O = 0 and
 *   lse = -inf. The merged result equals one softmax over the multiset
 *   union of the keys the patterns give the row.
 *
 * Layouts (all row-major, last index fastest):
 *   q, k, v, out, dout, dq, dk, dv : [B][N][H][d]
 *   lse                            : [B][H][N] float32, natural log
 * Element types: the unsuffixed entry points take bfloat16 tensors (stored as
 * 16-bit words) and compute in fp32 with bf16 tensor-core products; their
 * out is bf16 and the backward's gradients are fp32. The _f32 entry points
 * take and return float32 tensors and compute in plain fp32.
 *
 * Ownership: every tensor pointer is a DEVICE pointer owned by the caller;
 * the library keeps no reference after the call returns. w and r are HOST
 * arrays of npat ints, read before the call returns. The backward's
 * workspace is caller-owned device memory of at least
 * dilattn_bwd_workspace_size(...) bytes, 256-byte aligned; its contents on
 * entry do not matter and are garbage on return. Library-owned device
 * memory: one error word per device, the forward's scratch pool (below) and
 * the fixed array of dilattn_fwd_noalloc.
 *
 * Asynchrony: every compute entry point validates its arguments, enqueues
 * its kernels on `stream` and returns; faults during execution surface at the
 * caller's next synchronisation (ordinary CUDA semantics). Nothing throws
 * across the ABI. A status of DILATTN_ERR_CUDA leaves the CUDA error message
 * in dilattn_last_error().
 *
 * Constraints checked on every call (violations return
 * DILATTN_ERR_INVALID_ARG or DILATTN_ERR_UNSUPPORTED and launch nothing):
 *   B, N, H >= 1; 1 <= npat <= DILATTN_MAX_PATTERNS; w_i >= 1; r_i >= 1;
 *   causal in {0, 1}; B*N*H*d < 2^40; tensor pointers non-NULL and 16-byte
 *   aligned; outputs do not alias inputs; d in {64, 128}; the current device
 *   has compute capability 10.x.
 */
#ifndef DILATTN_H
#define DILATTN_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DILATTN_MAX_PATTERNS 16

enum dilattn_status {
  DILATTN_OK = 0,
  DILATTN_ERR_INVALID_ARG = 1,  /* bad shape, pointer, alignment or pattern */
  DILATTN_ERR_UNSUPPORTED = 2,  /* d not in {64, 128}, or device not CC 10.x */
  DILATTN_ERR_CUDA = 3,         /* a CUDA call or launch failed */
  DILATTN_ERR_WORKSPACE = 4,    /* workspace NULL, misaligned or too small */
  DILATTN_ERR_INTERNAL = 5      /* a kernel reported an internal failure */
};

/* Human-readable name of a status code (static string). */
const char* dilattn_status_string(int status);

/* Message of the last CUDA error this thread saw inside the library ("" if none). */
const char* dilattn_last_error(void);

/*
 * Forward: merged dilated attention (the whole method of the preamble; the
 * LongNet method description, gptget.net summary of arXiv 2307.02486,
 * "方法详解" bullets 1-3, and the shared-denominator merge of the DarcStar
 * commentary, third paragraph). Writes out [B][N][H][d] bf16 and, unless lse
 * is NULL, lse [B][H][N] fp32.
 *
 * The merge runs inside the forward: when a pattern has r = 1 (it keeps every
 * row), the tiles of that pattern finish each row, combining their own
 * online softmax with the stored partial results (normalised O_i and lse_i,
 * fp32) of the other patterns that keep the row, and write out and lse once;
 * the r = 1 pattern itself stores no partial. Without an r = 1 pattern every
 * pattern stores partials and a second kernel merges them. The partials live
 * in scratch of dilattn_fwd_scratch_size(...) bytes, which dilattn_fwd takes
 * stream-ordered from a memory pool the library creates per device on first
 * use (cudaMallocFromPoolAsync / cudaFreeAsync on `stream`; freed blocks stay
 * in the pool for the next call, so repeated calls map no new memory).
 * Callers that must not allocate use dilattn_fwd_noalloc.
 */
size_t dilattn_fwd_scratch_size(int B, int N, int H, int d, const int* w, const int* r,
                                int npat);
int dilattn_fwd(const void* q, const void* k, const void* v, void* out, float* lse,
                int B, int N, int H, int d, const int* w, const int* r, int npat, int causal,
                cudaStream_t stream);

/*
 * Forward for training: dilattn_fwd plus out_res [B][N][H][d] bf16, the
 * rounding residual bf16(O - out) of each output element, written by the
 * same fused epilogue. dilattn_bwd forms its row term D = rowsum(dout * O)
 * from out + out_res, i.e. from O to about 16 significant bits: D taken from
 * the bf16 out alone is off by sum_c dout_c (O_c - out_c), up to a few 1e-2,
 * which moves dq and dk by up to about 1e-2. out_res must not be NULL nor
 * overlap any other tensor argument.
 */
int dilattn_fwd_train(const void* q, const void* k, const void* v, void* out, void* out_res,
                      float* lse, int B, int N, int H, int d, const int* w, const int* r, int npat,
                      int causal, cudaStream_t stream);

/*
 * Forward with e4m3 q and k (FP8 variant; the gptget.net summary, "方法详解"
 * bullet 8, names quantisation among the engineering measures). q8, k8:
 * [B][N][H][d] e4m3 bytes holding q / q_scale and k / k_scale (per-tensor
 * scales > 0); v bf16. S = Q K^T runs on the FP8 tensor cores (kind::f8f6f4,
 * twice the bf16 rate) and is exact for the quantised inputs; P, V and the
 * PV product stay bf16, because an e4m3 P (3 mantissa bits) would cost far
 * more than the 2e-2 bound. d = 128 only: at d = 64 the forward is bound by
 * the exponentials, not by S. Results as dilattn_fwd for the inputs
 * q8 * q_scale, k8 * k_scale, v; scratch as in dilattn_fwd.
 */
int dilattn_fwd_fp8(const void* q8, const void* k8, const void* v, void* out, float* lse,
                    int B, int N, int H, int d, const int* w, const int* r, int npat, int causal,
                    float q_scale, float k_scale, cudaStream_t stream);

/*
 * Forward for callers that cannot allocate device memory: same arguments and
 * results as dilattn_fwd. Some callers have no way to get scratch memory: a
 * plugin handed only its input and output pointers by a host framework, a
 * server that reserves all device memory up front and forbids later
 * allocations, or code that must not risk the implicit device
 * synchronisation a cudaMalloc/cudaFree can bring. This entry point
 * allocates nothing, neither itself nor through any library: the forward's
 * scratch is a fixed array compiled into the library,
 * DILATTN_NOALLOC_SCRATCH_BYTES (64 MiB) large, which every device that
 * loads the library keeps reserved until the process exits. There is no
 * counterpart in the LongNet pages; it only changes where scratch lives.
 *
 * Limits and rules:
 *   - Problems whose dilattn_fwd_scratch_size(...) exceeds the array are
 *     rejected with DILATTN_ERR_WORKSPACE (dilattn_last_error() gives the two
 *     sizes); nothing is launched.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.
 *   - All calls on a device share the one array, and it keeps whatever the
 *     last call left there; the forward clears the part that must start at
 *     zero (its flags and ticket counter) itself, on `stream`. Calls that can
 *     overlap on the GPU -- on different streams, or from different host
 *     threads -- race on the array; the caller must order them, e.g. on one
 *     stream.
 *   - It returns out and lse like dilattn_fwd, not the out_res residual that
 *     dilattn_bwd takes: it serves inference; training uses
 *     dilattn_fwd_train.
 */
#define DILATTN_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)
int dilattn_fwd_noalloc(const void* q, const void* k, const void* v, void* out, float* lse,
                        int B, int N, int H, int d, const int* w, const int* r, int npat,
                        int causal, cudaStream_t stream);

/*
 * Sequence-parallel forward, one rank's part (LongNet's distributed
 * algorithm: the gptget.net summary of arXiv 2307.02486, "方法详解" bullet 5,
 * and the abstract's second contribution). The sequence of N = L * world
 * positions is split into world contiguous blocks of L; this rank holds
 * block `rank` of q, k, v ([B][L][H][d] bf16) and writes out ([B][L][H][d])
 * and lse ([B][H][L]) for its own rows, equal to the single-device
 * dilattn_fwd on the whole sequence restricted to those rows.
 *
 * A pattern with w <= L keeps its segments inside one block (L must be a
 * multiple of w) and runs locally. A pattern with w > L spans
 * min(w, N) / L ranks per segment (N a multiple of w unless w >= N; L a
 * multiple of r; L / r a multiple of 128): every rank of the segment packs
 * its kept rows of k and v (dilattn_pack_dilated: for head h the rows
 * (h mod r) + m r of its block, [B][L/r][H][d]), the ranks all-gather them
 * in rank order, and kg[i], vg[i] point to the gathered
 * [ranks][B][L/r][H][d] buffers of this rank's segment. Only those dilated
 * rows cross between ranks, never a full block. kg, vg may be NULL when no
 * pattern spans ranks. Scratch as in dilattn_fwd.
 *
 * Errors: DILATTN_ERR_INVALID_ARG for the argument errors of dilattn_fwd, a
 * rank outside [0, world), a split the rules above do not allow, a missing
 * or misaligned gathered buffer, or out / lse overlapping a gathered buffer
 * (the kernel reads those while it writes out and lse).
 */
int dilattn_fwd_seqpar(const void* q, const void* k, const void* v, void* out, float* lse,
                       int B, int L, int H, int d, const int* w, const int* r, int npat,
                       int causal, int rank, int world, const void* const* kg,
                       const void* const* vg, cudaStream_t stream);

/*
 * The rows a rank sends for a pattern of dilation r that spans ranks (the
 * dilated rows of LongNet's distributed algorithm, same passages as
 * dilattn_fwd_seqpar): buf[b][m][h][:] = x[b][(h mod r) + m r][h][:] for
 * m < L / r (x and buf bf16, device, 16-byte aligned, caller-owned; buf holds
 * B * (L / r) * H * d elements; L a multiple of r; d in {64, 128}).
 * Errors: DILATTN_ERR_INVALID_ARG for any of those violated or buf overlapping x.
 */
int dilattn_pack_dilated(const void* x, void* buf, int B, int L, int H, int d, int r,
                         cudaStream_t stream);

/*
 * Backward of dilattn_fwd_train (the full derivative of the merged function:
 * the merge weights depend on the scores and are differentiated, which
 * equals the gradient of one softmax over the multiset union of the keys
 * each row attends; DarcStar commentary, third paragraph). Given out,
 * out_res and lse from that forward and the output gradient dout (bf16,
 * [B][N][H][d]), writes the gradients of sum(O * dout): dq, dk, dv
 * [B][N][H][d] FLOAT32, the precision they are accumulated in (a caller
 * that keeps bf16 gradients rounds them). The probabilities are recomputed
 * from the saved lse; the row term D = rowsum(dout * O) is formed from
 * out + out_res. Workspace: D, the key-tile kernel's work counter and fp16
 * copies of q and k (the products with dS run in fp16), at least
 * dilattn_bwd_workspace_size(B, N, H, d) bytes, 256-byte aligned;
 * the workspace and dq, dk, dv must not overlap any input or each other.
 * Calls that share a workspace or gradient buffers must not overlap on the
 * GPU. d = 64 only (DILATTN_ERR_UNSUPPORTED otherwise; the fp32 entry point
 * covers d = 128).
 */
size_t dilattn_bwd_workspace_size(int B, int N, int H, int d);
int dilattn_bwd(const void* q, const void* k, const void* v, const void* out,
                const void* out_res, const float* lse, const void* dout, float* dq, float* dk,
                float* dv, int B, int N, int H, int d, const int* w, const int* r, int npat,
                int causal, void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * fp32 forward and backward: the same operation as dilattn_fwd / dilattn_bwd
 * (same passages), float32 tensors, no workspace, full fp32 FMA arithmetic
 * without TF32. Meant for small problems: each output row is computed by
 * one thread.
 */
int dilattn_fwd_f32(const float* q, const float* k, const float* v, float* out, float* lse,
                    int B, int N, int H, int d, const int* w, const int* r, int npat,
                    int causal, cudaStream_t stream);
int dilattn_bwd_f32(const float* q, const float* k, const float* v, const float* out,
                    const float* lse, const float* dout, float* dq, float* dk, float* dv,
                    int B, int N, int H, int d, const int* w, const int* r, int npat,
                    int causal, cudaStream_t stream);

/*
 * Row selection ("方法详解" bullets 1-3: segments of length w, every r-th row,
 * offset h mod r per head), as the attention kernels see it: sig [H][N]
 * (device, uint32) receives bit i at (h, n) when pattern i keeps row n for
 * head h.
 * It enumerates kept rows with the same segment/offset code the attention
 * kernels use to address their tiles, so it checks that code bit for bit.
 */
int dilattn_selection(uint32_t* sig, int N, int H, const int* w, const int* r, int npat,
                      cudaStream_t stream);

/*
 * Tracing hook. When both events are non-NULL, every later dilattn_fwd and
 * dilattn_bwd call made by the calling host thread records tile_begin on its
 * stream right before it launches its main tile kernel and tile_end right
 * after, so the caller can time that one kernel with cudaEventElapsedTime.
 * Passing NULL, NULL turns tracing off. The events stay owned by the caller
 * and must outlive the calls that record them.
 */
int dilattn_set_trace_events(cudaEvent_t tile_begin, cudaEvent_t tile_end);

/*
 * Reads and clears the library's device-side error word on the current
 * device after synchronising `stream`. *code receives 0 when no kernel
 * reported a failure, else the code of the last failure (1: a bounded wait
 * ran out). Every kernel launch carries its own tag, and its waits give up
 * early only on a failure of that same launch, so a failure that nobody has
 * read yet does not cut short the work of later calls; it stays readable
 * until this call clears it. The word's device address is looked up once
 * per device and cached: it does not survive cudaDeviceReset (nor does the
 * scratch of dilattn_fwd_noalloc).
 */
int dilattn_device_error(cudaStream_t stream, int* code);

/*
 * Self-test of the failure path (no counterpart in the LongNet pages). One
 * CTA with two warps: warp 0 waits on an mbarrier that nothing ever arrives
 * on, with a limit of limit_ns (1 .. 10^9); warp 1 waits on another such
 * barrier with the kernels' ordinary 4 s limit and must give up as soon as
 * warp 0 raises the CTA's abort flag. The kernel then returns, leaving code 1
 * in the device error word. result: device int[4], 16-byte aligned:
 * result[0], result[1] = 1 if warp 0's / warp 1's wait completed (neither may),
 * else 0; result[2], result[3] = the nanoseconds each waited (capped at 2e9).
 */
int dilattn_selftest_wait_timeout(unsigned long long limit_ns, int* result, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* DILATTN_H */

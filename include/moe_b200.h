/*
 * moe_b200.h — C ABI of the expert-routed MoE FFN layer for NVIDIA B200 (sm_100a).
 *
 * One call of the layer maps hidden states X [T, d] to the FFN output [T, d]:
 *   route    logits = X Wr^T (+ b) in fp32; per token the k largest logits, ties to
 *            the lower expert index, in rank order; gates = softmax over the k selected
 *            logits. (Qwen3.8-Flash-Next-Dual-GPU README, "Independent decode lane": the
 *            512-expert router uses a deterministic stable top-k; "Model artifact and
 *            memory placement": the router is kept in BF16/F32.)
 *   permute  an expert-major plan of the T*k assignments a = t*k + j: counts per expert,
 *            their exclusive scan, and a stable scatter (experts ascending, tokens
 *            ascending within an expert). (Same README, "Dedicated prefill lane", step 1;
 *            TandemLLM docs, "17 Qwen3.8-Flash-Next", §17.4: rows sorted by expert, one
 *            matrix product over each expert's rows.)
 *   grouped FFN  for every grouped row r of expert e: h = silu(Wg_e x) * (Wu_e x),
 *            y = Wd_e h, with group-quantised weights W = q * s (symmetric W4/W8, groups
 *            of 128 along K, BF16 scales: README, "Model artifact and memory placement").
 *            Unselected experts are never read (TandemLLM docs §17.4).
 *   combine  out_t = sum_{j<k} gate[t,j] * y[inv[t*k+j]] + y_shared[t], summed in that
 *            fixed order in fp32, rounded once to bf16, no atomics (README, "Dedicated
 *            prefill lane", step 5). The shared expert runs on every token with weight 1
 *            (TandemLLM docs Table 17.1: 10 routed and 1 shared run a token).
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers unless stated otherwise, 16-byte aligned,
 *     row-major, owned by the caller. The library never allocates device memory, never
 *     frees, and never synchronises the stream on the compute path.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = the legacy default stream).
 *   - Arguments are validated on the host before anything is enqueued; an invalid call
 *     returns a negative moe_status and enqueues nothing. No call throws across the ABI.
 *   - bf16 values are IEEE bfloat16 bit patterns (uint16).
 *   - Weight encodings (bank.fmt):
 *       MOE_W_BF16  W[e][n][k] bf16; scales unused (NULL).
 *       MOE_W_INT8  W[e][n][k] int8 (symmetric, code range -127..127), scales bf16
 *                   S[e][n][k / group].
 *       MOE_W_INT4  W[e][n][k / 8] uint32, 8 two's-complement nibbles per word along K,
 *                   element k at bits 4 * (k % 8) of word k / 8; scales as for int8.
 *       MOE_W_NVFP4 (routed bank only) NVFP4, the W4A4 variant of the layer (Anvil serving
 *                   benchmarks, "Qwen3.8 Flash Next", "Quantization boundary": ModelOpt
 *                   NVFP4 W4A4 on the routed experts, the shared expert kept BF16):
 *                   W[e][n][k / 2] uint8 of E2M1 codes, element k at bits 4 * (k % 2) of
 *                   byte k / 2; one E4M3 scale per 16 consecutive K values, stored in the
 *                   tensor-core layout that moe_nvfp4_pack_scales writes (group = 16);
 *                   one fp32 tensor scale per expert matrix in g_gate / g_up / g_down
 *                   ([n_exp] each). value = e2m1 * e4m3 * g. The activations entering the
 *                   routed experts (x, and h = silu(gate) * up rounded to fp32) are
 *                   quantised to NVFP4 per row at run time: g_row = amax / (6 * 448),
 *                   block scale = E4M3(amax_block / (6 g_row)), element =
 *                   E2M1(v / (block scale * g_row)), both nearest-even, every step an
 *                   IEEE fp32 operation. Such layers run on the FP4 tensor cores
 *                   (tcgen05.mma kind::mxf4nvf4) for every T; path must be AUTO or TC.
 *     gate and up are [n_exp][f][d] (N = f, K = d); down is [n_exp][d][f] (N = d, K = f).
 *     The two banks may use different encodings (e.g. an int8 shared expert beside int4
 *     routed experts); the grouped products then run once per bank. The single-kernel
 *     1-token path and the TMA GEMV path need int4 in both banks; other calls take the
 *     register-streaming GEMV or the tensor-core path.
 *   - Supported shapes: 1 <= T, d % 128 == 0, f % 128 == 0, 1 <= k <= min(E, 32),
 *     1 <= E <= 1024, group == 128 for the integer formats, shared.n_exp in {0, 1}.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_ABI_VERSION 2

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

typedef struct CUstream_st* moe_stream_t; /* identical to cudaStream_t */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = -1, /* a pointer, size, alignment or shape is not accepted   */
  MOE_ERR_UNSUPPORTED = -2, /* a valid request the library does not implement       */
  MOE_ERR_CUDA = -3,        /* a CUDA runtime call failed (launch or attribute)       */
  MOE_ERR_TIMEOUT = -4,     /* a bounded device-side wait gave up (device status)     */
  MOE_ERR_WORKSPACE = -5,   /* workspace NULL, misaligned or smaller than required    */
  MOE_ERR_DEVICE = -6,      /* a device-side check failed (see moe_device_status)     */
  MOE_ERR_TOO_LARGE = -7    /* the request needs more than the library's built-in scratch */
} moe_status;

typedef enum { MOE_W_BF16 = 16, MOE_W_INT8 = 8, MOE_W_INT4 = 4, MOE_W_NVFP4 = 41 } moe_wfmt;

/* Which kernels run. AUTO picks the single-kernel layer (FUSED) for 1-token calls with
 * int4 banks when the device fits it, the split-K GEMV kernels for other calls of 1..32
 * rows, and the tensor-core (tcgen05) grouped GEMMs from 33 rows up. Up to 32 rows, AUTO is
 * row-invariant: a token's output (and its routing) is the same bits whether it is called
 * alone or among up to 32 rows, in any position (the single-kernel layer and the GEMV
 * kernels share one arithmetic order; TandemLLM docs, "17 Qwen3.8-Flash-Next", §17.3).
 * TC asks for the tensor cores at any T (not row-invariant with the 1-token layer). FUSED asks for the single-kernel layer and returns MOE_ERR_UNSUPPORTED
 * from moe_layer_forward when the call does not fit it; the stage entry points (moe_route ...
 * moe_combine) treat FUSED like GEMV. NVFP4 layers run on the FP4 tensor cores for every T. */
typedef enum { MOE_PATH_AUTO = 0, MOE_PATH_GEMV = 1, MOE_PATH_TC = 2, MOE_PATH_FUSED = 3 } moe_path;

/* One expert bank of n_exp experts (the routed bank has n_exp = E; the shared bank has
 * n_exp = 0 or 1). Pointers are device pointers; experts are contiguous, expert e's
 * slice starts at e * (N * K * bits / 8) bytes. */
typedef struct {
  int32_t fmt;   /* moe_wfmt */
  int32_t group; /* 128 for MOE_W_INT8 / MOE_W_INT4, 16 for MOE_W_NVFP4; ignored for bf16 */
  int32_t n_exp;
  int32_t reserved;
  const void* w_gate; /* [n_exp][f][d] encoded */
  const void* w_up;   /* [n_exp][f][d] encoded */
  const void* w_down; /* [n_exp][d][f] encoded */
  const void* s_gate; /* bf16 [n_exp][f][d / group], packed E4M3 (NVFP4), or NULL (bf16) */
  const void* s_up;   /* bf16 [n_exp][f][d / group], packed E4M3 (NVFP4), or NULL */
  const void* s_down; /* bf16 [n_exp][d][f / group], packed E4M3 (NVFP4), or NULL */
  const float* g_gate; /* NVFP4 only: fp32 [n_exp] tensor scales (NULL otherwise) */
  const float* g_up;
  const float* g_down;
} moe_bank;

/* The layer: shapes, router and the two banks. Read by every call; not retained. */
typedef struct {
  int32_t T, d, f, E, k;
  int32_t path;              /* moe_path */
  const void* router_w;      /* bf16 [E][d] */
  const float* router_bias;  /* fp32 [E] added to the logits, or NULL */
  moe_bank routed;           /* n_exp == E */
  moe_bank shared;           /* n_exp == 0 (no shared expert) or 1 */
} moe_layer;

/* ABI version of the loaded library (MOE_ABI_VERSION). */
MOE_API int32_t moe_abi_version(void);

/* Human-readable name of a status code. Never NULL; the string is static. */
MOE_API const char* moe_status_str(int32_t status);

/* Host-side validation of a layer descriptor (no CUDA call is made).
 * Returns MOE_OK or MOE_ERR_INVALID_ARG / MOE_ERR_UNSUPPORTED. */
MOE_API moe_status moe_validate(const moe_layer* L);

/* Bytes of device workspace every call on this layer needs (0 if L is invalid).
 * The workspace is caller-owned, 256-byte aligned, and may be reused between calls
 * that are ordered on one stream; concurrent calls need separate workspaces. Fill it with
 * zeros before its first use (cudaMemset): the calls keep the counters at its start at zero
 * from one call to the next. */
MOE_API size_t moe_workspace_size(const moe_layer* L);

/* Route: topk_idx int32 [T][k] (expert ids, rank order) and topk_w fp32 [T][k]
 * (gates, each row sums to 1). x: bf16 [T][d]. */
MOE_API moe_status moe_route(const moe_layer* L, const void* x, int32_t* topk_idx, float* topk_w,
                     void* ws, size_t ws_bytes, moe_stream_t stream);

/* Permute: from topk_idx [T][k], writes expert_offsets int32 [E + 1] (exclusive scan of
 * the per-expert counts; offsets[E] = T * k), perm int32 [T * k] (perm[r] = assignment
 * t * k + j at grouped row r) and inv int32 [T * k] (inv[t * k + j] = its grouped row). */
MOE_API moe_status moe_permute(const moe_layer* L, const int32_t* topk_idx, int32_t* expert_offsets,
                       int32_t* perm, int32_t* inv, void* ws, size_t ws_bytes,
                       moe_stream_t stream);

/* Grouped FFN over the plan: y_assign fp32 [T * k][d] in grouped row order (row r is
 * expert e's output for assignment perm[r], e such that offsets[e] <= r < offsets[e+1]),
 * and y_shared fp32 [T][d] (the shared expert on every token; may be NULL only when
 * shared.n_exp == 0). x: bf16 [T][d]. */
MOE_API moe_status moe_grouped_ffn(const moe_layer* L, const void* x, const int32_t* expert_offsets,
                           const int32_t* perm, float* y_assign, float* y_shared, void* ws,
                           size_t ws_bytes, moe_stream_t stream);

/* Combine: out bf16 [T][d] = sum_{j<k} topk_w[t][j] * y_assign[inv[t*k+j]] (+ y_shared[t]),
 * accumulated in fp32 in the order j = 0..k-1, then the shared term; one rounding. */
MOE_API moe_status moe_combine(const moe_layer* L, const float* y_assign, const float* y_shared,
                       const int32_t* inv, const float* topk_w, void* out,
                       moe_stream_t stream);

/* The whole layer in one call: out bf16 [T][d] from x bf16 [T][d]. The optional outputs
 * (topk_idx [T][k], topk_w [T][k], expert_offsets [E+1], perm [T*k]) are written when
 * non-NULL. Intermediates live in the workspace. */
MOE_API moe_status moe_layer_forward(const moe_layer* L, const void* x, void* out, int32_t* topk_idx,
                             float* topk_w, int32_t* expert_offsets, int32_t* perm, void* ws,
                             size_t ws_bytes, moe_stream_t stream);

/* Stage marks for profiling: the same computation as moe_layer_forward, and each non-NULL
 * entry of `marks` (cudaEvent_t handles created by the caller) is recorded on `stream`:
 * marks[0] before the first kernel, marks[1] after routing, marks[2] after the plan,
 * marks[3] after the gate/up kernel, marks[4] after the down kernel, marks[5] after the
 * combine. n_marks may be smaller than MOE_N_MARKS; missing entries are skipped. */
#define MOE_N_MARKS 6
MOE_API moe_status moe_layer_forward_marked(const moe_layer* L, const void* x, void* out,
                                    int32_t* topk_idx, float* topk_w, int32_t* expert_offsets,
                                    int32_t* perm, void* ws, size_t ws_bytes,
                                    moe_stream_t stream, void* const* marks, int32_t n_marks);

/* Number of kernels moe_layer_forward enqueues for this descriptor (0 if L is invalid).
 * Host-side only; it may query the current device's multiprocessor count (cached). */
MOE_API int32_t moe_launches_per_call(const moe_layer* L);

/* Reads the device status word kept in the workspace (synchronises `stream`), writes
 * the code to *code (MOE_OK, MOE_ERR_TIMEOUT or MOE_ERR_DEVICE) and clears it. */
MOE_API moe_status moe_device_status(const moe_layer* L, void* ws, size_t ws_bytes, int32_t* code,
                             moe_stream_t stream);

/* Where a MOE_ERR_TIMEOUT came from: the site of the first bounded device-side wait that gave
 * up since the last read (0: none), read from the workspace and cleared (synchronises
 * `stream`). Sites: 1 fused routing grid barrier, 2 fused routing test hold; 10..18 integer/
 * bf16 tensor-core GEMMs (10 scale buffer free, 11 weight stage free, 12 accumulator free,
 * 13 scales landed, 14 weight stage landed, 15 operand stage free, 16 activation stage landed,
 * 17 activation stage free (producer), 18 accumulator full); 20..25 single-kernel 1-token
 * layer (20 router rows landed, 21 gate/up tile landed, 22 first grid barrier, 23 second grid
 * barrier, 24 down unit landed, 25 h rows landed); 30 TMA GEMV stage free, 31 TMA GEMV stage
 * landed; 40..42 NVFP4 GEMMs (40 stage free, 41 accumulator free or stage landed, 42
 * accumulator full). */
MOE_API moe_status moe_device_wait_site(const moe_layer* L, void* ws, size_t ws_bytes,
                                        int32_t* site, moe_stream_t stream);

/* Failure injection, for tests of the error path: sets (hold != 0) or clears (hold == 0)
 * the hold word in the workspace's synchronisation block, with a wait budget in SM clock
 * cycles (0 = the library's normal bound of about two seconds). While the word is set, the
 * single-kernel 1-token layer (at its first grid barrier) and the fused routing kernel of
 * calls of up to 32 tokens (after its ticket barrier) wait for the word to return to zero,
 * which nothing does during a call: the wait runs out after the budget, the kernel records
 * MOE_ERR_TIMEOUT in the status word (read by moe_device_status), drains its copies and
 * returns, exactly as when a peer never arrives. Nothing hangs and nothing faults. The
 * words are written with an asynchronous copy on `stream` (not for use during capture).
 * Clear the word (or use a fresh workspace) before normal use. */
MOE_API moe_status moe_test_inject_hold(const moe_layer* L, void* ws, size_t ws_bytes,
                                        int32_t hold, int32_t budget_cycles,
                                        moe_stream_t stream);

/* For callers that cannot allocate device memory. Some callers have no way to call
 * cudaMalloc when the layer runs: code running inside a stream-ordered region whose
 * allocator is owned by someone else, plug-ins that are handed a stream but no allocator,
 * or processes with a fixed device-memory budget that was reserved up front. This entry
 * point runs the same layer as moe_layer_forward (same kernels, same result) but keeps
 * every intermediate in a scratch buffer that lives inside the library itself: a
 * 16 MiB array in device memory, part of the library's image on every GPU that loads it
 * and held until the process exits. It allocates nothing and frees nothing.
 *
 *   - Limit: the call's moe_workspace_size(L) must be at most MOE_STATIC_SCRATCH_BYTES
 *     (16 MiB; it covers decode and verify calls of up to 32 tokens at d <= 4096,
 *     f <= 2048, E <= 1024, k <= 16). Larger requests return MOE_ERR_TOO_LARGE and enqueue
 *     nothing.
 *   - The first call on a device looks up the buffer's device address (once per device);
 *     make that first call before capturing a stream into a CUDA graph.
 *   - Every call on a device shares the one buffer, and it keeps the previous call's
 *     contents (the call clears the words that must start at zero, except the status
 *     word, which moe_static_device_status reads and clears). Calls that can run at
 *     the same time on one device (different streams, or different host threads without
 *     ordering) race on it and give wrong results; order them on one stream.
 *   - x and out as for moe_layer_forward; the routing outputs are not returned.
 * This entry point has no counterpart in the pages the layer follows; it is a deployment
 * aid of this library. */
#define MOE_STATIC_SCRATCH_BYTES (16u << 20)
MOE_API moe_status moe_layer_forward_static(const moe_layer* L, const void* x, void* out,
                                            moe_stream_t stream);

/* The device status word of the built-in scratch used by moe_layer_forward_static on the
 * current device (the counterpart of moe_device_status for that entry point): synchronises
 * `stream`, writes MOE_OK, MOE_ERR_TIMEOUT or MOE_ERR_DEVICE to *code and clears the word.
 * A static call leaves the word as its kernels set it (it does not clear it), so an error
 * of any call since the last read is reported here. Allocates nothing. Like the first static
 * call, the first call of this function on a device looks up the buffer's address. */
MOE_API moe_status moe_static_device_status(int32_t* code, moe_stream_t stream);

/* Block scales of an NVFP4 bank in the layout its kernels read. `src` holds one E4M3 byte per
 * 16 consecutive K values of each row, row-major: uint8 [n_mats][rows][K / 16] (the natural
 * order). `dst` (same size, caller-owned, 16-byte aligned) receives, for each matrix, each
 * tile of 128 rows and each step of 64 K values, one 512-byte block in which the scale of row
 * 128 * tile + 32 * q + i (i < 32, q < 4) for K values 64 * step + 16 * j .. +15 (j < 4) sits at
 * byte 16 * i + 4 * q + j: the order in which the tensor core takes a 128-row operand's scales
 * into tensor memory (tcgen05.cp, 32 lanes x 128 bits, repeated in the four lane quarters).
 * Call once per bank when the weights are loaded; pass dst as the bank's s_* pointer.
 * rows % 128 == 0, K % 64 == 0, n_mats >= 1. Enqueued on `stream`; src and dst must not
 * overlap. Returns MOE_ERR_INVALID_ARG for a bad size or pointer. */
MOE_API moe_status moe_nvfp4_pack_scales(const void* src, void* dst, int32_t n_mats, int32_t rows,
                                         int32_t K, moe_stream_t stream);

/* NVFP4 quantisation of fp32 rows, as the layer applies it to the activations entering NVFP4
 * routed experts: per row, g = amax / (6 * 448) (fp32 [rows]); per block of 16 values the E4M3
 * code of amax_block / (6 g), nearest even, saturating at 448 (uint8 [rows][K / 16], natural
 * order); the E2M1 codes of v / (e4m3 * g), nearest even, saturating at 6 (uint8
 * [rows][K / 2], element k at bits 4 * (k % 2) of byte k / 2); each step one IEEE fp32
 * operation; a zero row gives zero codes. v: fp32 [rows][K], K % 16 == 0, K <= 8192, rows >= 1;
 * every pointer 16-byte aligned (g: 4). Enqueued on `stream`. */
MOE_API moe_status moe_nvfp4_quantize_rows(const float* v, int32_t rows, int32_t K, void* codes,
                                           void* scales, float* g, moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */

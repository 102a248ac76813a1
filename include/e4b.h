/*
 * e4b.h -- C ABI of libe4b: the routed Mixture-of-Experts expert layer run
 * directly on NF4-packed fused expert stacks, on one NVIDIA B200 (sm_100a).
 *
 * The operations follow the pages this library is written from:
 *   - fused stacks gate_up_proj [E, 2I, H] and down_proj [E, H, I]
 *     ("Why does load_in_4bit still OOM on a Mixture-of-Experts model?",
 *     section "Why it happens");
 *   - 4-bit NF4 storage with blocks of 64 that never cross an expert boundary
 *     (same page, "Which project solves it"; experts4bit-qlora 0.22.0,
 *     "Install": the fast path takes NF4 with blocksize 64 only);
 *   - sorting token/expert pairs into per-expert groups (experts4bit-qlora
 *     0.22.0, "Which training path?");
 *   - one grouped GEMM launch that decodes the nibbles in registers with fp32
 *     accumulation and materialises no bf16 expert tensor (Solutions -- one
 *     page per problem, the grouped-nf4-gemm row on gemm_4bit_grouped);
 *   - the SwiGLU expert MLP ("Scope") and the per-expert LoRA delta added
 *     before the activation (Solutions page, the ExpertsLoRA row; r=8,
 *     alpha=16 in "Quickstart").
 *
 * Conventions for every call
 *   - Pointers to tensors are DEVICE pointers unless a comment says otherwise.
 *     The caller allocates and owns every buffer, workspaces included; the
 *     library never allocates, frees or synchronises on these calls.
 *   - Tensors are contiguous, row-major and 16-byte aligned (base address),
 *     except where a leading dimension is passed.
 *   - bf16 data is passed as raw 16-bit patterns (uint16_t).
 *   - Calls are stream-ordered on `stream` (a cudaStream_t; NULL is the legacy
 *     default stream).  The four calls of the layer (quantise, route/permute,
 *     grouped GEMM, forward) read no device data back to the host and can be
 *     captured in a CUDA graph.
 *   - Arguments are checked on the host before anything is launched.  A bad
 *     argument returns E4B_ERR_INVALID_ARGUMENT, a shape or device the kernels
 *     do not support returns E4B_ERR_UNSUPPORTED, a workspace that is too small
 *     returns E4B_ERR_WORKSPACE, and a failed launch returns E4B_ERR_CUDA.
 *     e4b_last_error() then names the argument or the CUDA error.  Nothing
 *     falls back silently to another path: the path that ran is reported by
 *     e4b_last_path().
 *   - Device data that breaks a documented invariant (offsets that are not
 *     non-decreasing, indices out of range) cannot be checked on the host; the
 *     kernels clamp such values so that no access leaves the buffers, and the
 *     affected outputs are unspecified.
 *   - Workspaces are 16-byte aligned like every other buffer.  The first 4
 *     bytes of a workspace of e4b_grouped_nf4_gemm() or e4b_moe_expert_forward()
 *     are an error word: a kernel whose bounded wait (2 s) gives up writes a
 *     nonzero E4B_KERNEL_ERR_* code there (the first code wins) and returns,
 *     and the output of that call is unspecified.  Nothing clears the word, so
 *     allocate workspaces zeroed (or clear them with
 *     e4b_workspace_clear_error()) and read it with e4b_workspace_error().
 */
#ifndef E4B_H_
#define E4B_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define E4B_VERSION 3

#if defined(__GNUC__)
#define E4B_API __attribute__((visibility("default")))
#else
#define E4B_API
#endif

typedef enum {
  E4B_OK = 0,
  E4B_ERR_INVALID_ARGUMENT = 1,
  E4B_ERR_UNSUPPORTED = 2, /* shape, dtype or device (not sm_100) */
  E4B_ERR_WORKSPACE = 3,   /* workspace smaller than the size query returns */
  E4B_ERR_CUDA = 4         /* a CUDA runtime call or a launch failed */
} e4b_status;

typedef enum { E4B_F32 = 0, E4B_BF16 = 1 } e4b_dtype;

typedef enum {
  E4B_EPI_NONE = 0,  /* out = A_rows . W^T                                  */
  E4B_EPI_SWIGLU = 1 /* y = A_rows . W^T (+ LoRA); out = SiLU(y[:, :N/2]) * y[:, N/2:] */
} e4b_epilogue;

/*
 * The 4-bit storage of a packed stack: which 16-entry codebook its codes
 * index.  Both share the layout of e4b_quantize_stack() (blocks of 64, fp32
 * absmax, two codes per byte, the lower-index element in the high nibble).
 * Source: experts4bit-qlora 0.22.0, opening section and "Scope" (the storage
 * modes nf4 and fp4 of one fused stack, with NF4 the more accurate).
 */
typedef enum {
  E4B_QUANT_NF4 = 0, /* the NF4 table of the QLoRA paper, ascending, entry 7 = 0 */
  E4B_QUANT_FP4 = 1  /* e2m1 codes over 6: code c = (-1)^(c>>3) * m[c & 7] / 6 with
                        m = 0, 0.5, 1, 1.5, 2, 3, 4, 6 (codes 0 and 8 are zero) */
} e4b_quant_type;

/* Which implementation e4b_moe_expert_forward_path() runs. */
typedef enum {
  E4B_PATH_AUTO = 0,    /* small token counts -> DECODE, otherwise GROUPED */
  E4B_PATH_DECODE = 1,  /* fused split-row GEMV over the touched experts only */
  E4B_PATH_GROUPED = 2  /* grouped tensor-core GEMMs + combine */
} e4b_path;

typedef struct CUstream_st* e4b_stream; /* identical to cudaStream_t */

/* Human-readable name of a status code (static string). */
E4B_API const char* e4b_status_string(e4b_status s);

/* Detail of the last failing call on this host thread ("" if none). */
E4B_API const char* e4b_last_error(void);

/* Name of the kernel path the last successful call on this host thread
 * launched, e.g. "quantize", "route.small", "gemm.tc", "forward.decode". */
E4B_API const char* e4b_last_path(void);

/* Error word codes (see the conventions above). */
#define E4B_KERNEL_ERR_NONE 0
#define E4B_KERNEL_ERR_WAIT_FULL 1  /* a consumer waited in vain for its input tile */
#define E4B_KERNEL_ERR_WAIT_EMPTY 2 /* a producer waited in vain for a free stage */
#define E4B_KERNEL_ERR_WAIT_DRAIN 3 /* a CTA gave up waiting for its own copies */
#define E4B_KERNEL_ERR_GRID_BARRIER 4 /* a CTA of the decode kernel gave up waiting for the others */

/* Reads the error word of `workspace` into *code.  Synchronises the device
 * first (a diagnostic call, not for the hot path or a graph capture).  This
 * call and the next leave e4b_last_path() and e4b_last_launches() as the
 * previous call set them. */
E4B_API e4b_status e4b_workspace_error(const void* workspace, int32_t* code);

/* Sets the error word of `workspace` to E4B_KERNEL_ERR_NONE, ordered on `stream`. */
E4B_API e4b_status e4b_workspace_clear_error(void* workspace, e4b_stream stream);

/* E4B_VERSION of the built library. */
E4B_API int e4b_version(void);

/* Number of kernels the last call on this host thread launched. */
E4B_API int e4b_last_launches(void);

/*
 * Kernel timing for benchmarks and profiling (host thread local).
 * e4b_timing_enable(1) clears earlier records and, until e4b_timing_enable(0),
 * brackets every kernel the library launches on this thread with a pair of
 * CUDA events recorded on the launch stream (events are created on first use
 * and reused).  e4b_timing_kernels() counts the distinct kernel names
 * recorded; e4b_timing_get(i, ...) waits for the events of kernel name i and
 * returns its total elapsed milliseconds and launch count.  Not for use inside
 * a CUDA graph capture.
 */
E4B_API e4b_status e4b_timing_enable(int on);
E4B_API int e4b_timing_kernels(void);
E4B_API e4b_status e4b_timing_get(int i, const char** name, double* total_ms, int* launches);

/*
 * a1 -- NF4 quantisation of a fused expert stack.
 * Source: "Why does load_in_4bit still OOM on a Mixture-of-Experts model?",
 * "Which project solves it" (blocks never cross an expert boundary).
 *
 * W        [E, N, K] row-major, fp32 (w_dtype E4B_F32) or bf16 (E4B_BF16).
 * packed   [E, N*K/2] uint8 out.  Each expert is flattened row-major and cut
 *          into blocks of 64 consecutive elements; byte j holds the codes of
 *          elements 2j (high nibble) and 2j+1 (low nibble).
 * absmax   [E, N*K/64] fp32 out: the largest |w| of each block.
 * Each code is the nearest entry of the 16-entry NF4 codebook (QLoRA table,
 * ascending, entry 7 = 0) to s = w / absmax computed as one IEEE fp32
 * division; a value exactly between two entries takes the lower index; an
 * all-zero block stores absmax 0 and code 7.  Bit-exact by construction.
 * Requires blocksize == 64, E >= 1, N >= 1, K >= 1, (N*K) % 64 == 0.
 * Non-finite inputs give unspecified codes (no fault).
 */
E4B_API e4b_status e4b_nf4_quantize_stack(const void* W, e4b_dtype w_dtype, int64_t E, int64_t N,
                                  int64_t K, int blocksize, uint8_t* packed, float* absmax,
                                  e4b_stream stream);

/*
 * The same quantiser for either 4-bit storage (e4b_quant_type).  With
 * E4B_QUANT_NF4 it is e4b_nf4_quantize_stack().  With E4B_QUANT_FP4 each code
 * is the one whose value is nearest to s = w / absmax (one IEEE fp32
 * division) in exact arithmetic; a value exactly between two values takes the
 * smaller; zero is code 0 (code 8 is never written); an all-zero block stores
 * absmax 0 and code 0.  Bit-exact by construction.  Same requirements as
 * above; a quant_type other than the two is E4B_ERR_INVALID_ARGUMENT.
 */
E4B_API e4b_status e4b_quantize_stack(const void* W, e4b_dtype w_dtype, int64_t E, int64_t N, int64_t K,
                                      int blocksize, e4b_quant_type quant_type, uint8_t* packed,
                                      float* absmax, e4b_stream stream);

/*
 * a2 + a3 -- router top-k and the token/expert permutation.
 * Source: experts4bit-qlora 0.22.0, "Which training path?" (sort the
 * token/expert pairs, run the groups); routing "softmax top-k renormalised".
 *
 * logits          [M, E] fp32.
 * topk_ids        [M, k] int32 out: per token, experts ordered by (logit
 *                 descending, index ascending); slot j = the j-th.
 * topk_w          [M, k] fp32 out: renormalize != 0: softmax over the k
 *                 selected logits; renormalize == 0: the full softmax over E
 *                 evaluated at the selected experts.
 * expert_offsets  [E+1] int32 out: first permuted position of each expert;
 *                 expert_offsets[E] = M*k.
 * perm            [M*k] int32 out: flat slots f = t*k + j in a stable sort
 *                 by expert id.
 * inv_perm        [M*k] int32 out: inv_perm[perm[p]] = p.
 * workspace       device scratch of e4b_moe_route_permute_workspace_size()
 *                 bytes (may be NULL when that size is 0).
 * Requires M >= 0, 1 <= E <= 1024, 1 <= k <= min(E, 32).  M == 0 writes only
 * expert_offsets (all zero).  ids and perm are bit-exact; weights use expf.
 * NaN logits give unspecified (in-range) ids.
 */
E4B_API size_t e4b_moe_route_permute_workspace_size(int64_t M, int64_t E, int k);
E4B_API e4b_status e4b_moe_route_permute(const float* logits, int64_t M, int64_t E, int k,
                                 int renormalize, int32_t* topk_ids, float* topk_w,
                                 int32_t* expert_offsets, int32_t* perm, int32_t* inv_perm,
                                 void* workspace, size_t workspace_bytes, e4b_stream stream);

/*
 * a4..a7 -- one grouped GEMM over E expert groups on NF4-packed weights.
 * Source: Solutions -- one page per problem, the grouped-nf4-gemm row
 * (gemm_4bit_grouped: one launch, nibbles decoded in registers, fp32
 * accumulation).
 *
 * Row p (0 <= p < total_rows) belongs to the group e with
 * expert_offsets[e] <= p < expert_offsets[e+1] and computes
 *     y[p, :] = A[row_index[p], :] . W_e^T                      (N values)
 *     y[p, :] += lora_scale * (A[row_index[p], :] . lora_A[e]^T) . lora_B[e]^T
 * where W_e = codebook[q] * absmax is expert e's [N, K] NF4 matrix.
 *
 * A               [a_rows, lda] bf16 (lda >= K, in elements, lda % 8 == 0).
 * row_index       [total_rows] int32 indices into A, or NULL for p itself.
 * expert_offsets  [E+1] int32, non-decreasing, expert_offsets[E] == total_rows.
 * packed, absmax  [E, N*K/2] uint8 and [E, N*K/64] fp32 (e4b_nf4_quantize_stack).
 * lora_A, lora_B  [E, r, K] and [E, N, r] bf16, or both NULL (no adapter);
 *                 16-byte aligned like every other tensor.
 * epi             E4B_EPI_NONE: out[p, n] = y[p, n], n < N.
 *                 E4B_EPI_SWIGLU: out[p, n] = SiLU(y[p, n]) * y[p, N/2 + n],
 *                 n < N/2 (gate = first half of the rows, up = second half).
 * out             [total_rows, N or N/2] of out_dtype.
 * Requires K % 64 == 0, N % 64 == 0, 0 <= r <= 16, total_rows < 2^31.
 * workspace       e4b_grouped_nf4_gemm_workspace_size() bytes: an error word,
 *                 the LoRA products x . lora_A^T (total_rows x r fp32) and room
 *                 for the routed rows gathered in order (total_rows x K bf16),
 *                 which the tensor-core kernel reads as contiguous tiles when
 *                 row_index is given.  0 bytes (NULL allowed) when total_rows == 0.
 * Groups with no rows cost nothing and write nothing.
 */
E4B_API size_t e4b_grouped_nf4_gemm_workspace_size(int64_t total_rows, int64_t N, int64_t K, int r);
E4B_API e4b_status e4b_grouped_nf4_gemm(const uint16_t* A, int64_t a_rows, int64_t lda,
                                const int32_t* row_index, const int32_t* expert_offsets,
                                int64_t E, int64_t total_rows, const uint8_t* packed,
                                const float* absmax, int64_t N, int64_t K,
                                const uint16_t* lora_A, const uint16_t* lora_B, int r,
                                float lora_scale, e4b_epilogue epi, void* out,
                                e4b_dtype out_dtype, void* workspace, size_t workspace_bytes,
                                e4b_stream stream);

/* e4b_grouped_nf4_gemm() on a stack of either 4-bit storage: W_e =
 * codebook(quant_type)[q] * absmax.  Same arguments, workspace and
 * requirements; e4b_grouped_nf4_gemm() is this call with E4B_QUANT_NF4. */
E4B_API e4b_status e4b_grouped_4bit_gemm(const uint16_t* A, int64_t a_rows, int64_t lda,
                                 const int32_t* row_index, const int32_t* expert_offsets,
                                 int64_t E, int64_t total_rows, const uint8_t* packed,
                                 const float* absmax, e4b_quant_type quant_type, int64_t N,
                                 int64_t K, const uint16_t* lora_A, const uint16_t* lora_B, int r,
                                 float lora_scale, e4b_epilogue epi, void* out,
                                 e4b_dtype out_dtype, void* workspace, size_t workspace_bytes,
                                 e4b_stream stream);

/*
 * Backward through the frozen base -- the input gradient of the grouped NF4
 * GEMM above, in one launch over all groups.
 * Source: experts4bit-qlora 0.22.0, "Which training path?" (the backward's
 * dgrad runs as one launch instead of a per-expert decode loop; the frozen
 * base is decoded again from the packed bytes, never kept dequantised).
 *
 * Row p (0 <= p < total_rows) of group e computes
 *     dx[p, :] = dY[row_index[p], :] . W_e                       (K values)
 *     dx[p, :] += lora_scale * (dY[row_index[p], :] . lora_B[e]) . lora_A[e]
 * with W_e expert e's [N, K] NF4 matrix as in e4b_grouped_nf4_gemm(): for a
 * forward y = a . W_e^T (+ adapter), dx is the gradient of <dY, y> by a.
 *
 * dY              [dy_rows, lddy] bf16 (lddy >= N, lddy % 8 == 0).
 * row_index       [total_rows] int32 indices into dY, or NULL for p itself.
 * expert_offsets, packed, absmax, lora_A, lora_B: as in e4b_grouped_nf4_gemm().
 * out             [total_rows, K] of out_dtype.
 * Requires K % 64 == 0, N % 64 == 0, 0 <= r <= 16, total_rows < 2^31.
 * workspace       e4b_grouped_nf4_gemm_dgrad_workspace_size() bytes: an error
 *                 word and the products dY . lora_B (total_rows x r fp32).
 *                 0 bytes (NULL allowed) when total_rows == 0.
 * Groups with no rows cost nothing and write nothing.
 */
E4B_API size_t e4b_grouped_nf4_gemm_dgrad_workspace_size(int64_t total_rows, int64_t N, int64_t K, int r);
E4B_API e4b_status e4b_grouped_nf4_gemm_dgrad(const uint16_t* dY, int64_t dy_rows, int64_t lddy,
                                      const int32_t* row_index, const int32_t* expert_offsets,
                                      int64_t E, int64_t total_rows, const uint8_t* packed,
                                      const float* absmax, int64_t N, int64_t K,
                                      const uint16_t* lora_A, const uint16_t* lora_B, int r,
                                      float lora_scale, void* out, e4b_dtype out_dtype,
                                      void* workspace, size_t workspace_bytes, e4b_stream stream);

/* e4b_grouped_nf4_gemm_dgrad() on a stack of either 4-bit storage; same
 * arguments, workspace and requirements. */
E4B_API e4b_status e4b_grouped_4bit_gemm_dgrad(const uint16_t* dY, int64_t dy_rows, int64_t lddy,
                                       const int32_t* row_index, const int32_t* expert_offsets,
                                       int64_t E, int64_t total_rows, const uint8_t* packed,
                                       const float* absmax, e4b_quant_type quant_type, int64_t N,
                                       int64_t K, const uint16_t* lora_A, const uint16_t* lora_B,
                                       int r, float lora_scale, void* out, e4b_dtype out_dtype,
                                       void* workspace, size_t workspace_bytes, e4b_stream stream);

/*
 * The adapter's gradients of one grouped projection (backward of the
 * per-expert LoRA delta over the frozen NF4 base).
 * Source: Solutions -- one page per problem, the ExpertsLoRA row (a per-expert
 * low-rank delta before each routed expert's activation, trained over the
 * frozen stack); experts4bit-qlora 0.22.0, "Which training path?".
 *
 * For the forward y_p = x_p . W_e^T + s (x_p . A_e^T) . B_e^T of
 * e4b_grouped_nf4_gemm() (x_p = x[row_index[p]]) and the gradient da of its
 * output rows (group order, [total_rows, ldda]):
 *     dB_e = s * sum_{p in e} da_p^T (x_p . A_e^T)          [N, r] fp32
 *     dA_e = s * sum_{p in e} (da_p . B_e)^T x_p            [r, K] fp32
 * summed over each group's rows in order (deterministic); experts without rows
 * get zeros.  x [x_rows, ldx] bf16 (ldx >= K, ldx % 8 == 0), da bf16,
 * lora_A [E, r, K], lora_B [E, N, r] bf16, dA [E, r, K], dB [E, N, r] fp32.
 * Requires K % 64 == 0, N % 64 == 0, 1 <= r <= 16.
 * workspace       e4b_grouped_lora_grads_workspace_size() bytes: an error
 *                 word and the products x . A^T and da . B (total_rows x r fp32 each).
 */
E4B_API size_t e4b_grouped_lora_grads_workspace_size(int64_t total_rows, int r);
E4B_API e4b_status e4b_grouped_lora_grads(const uint16_t* x, int64_t x_rows, int64_t ldx,
                                  const int32_t* row_index, const int32_t* expert_offsets,
                                  int64_t E, int64_t total_rows, const uint16_t* da, int64_t ldda,
                                  int64_t N, int64_t K, const uint16_t* lora_A,
                                  const uint16_t* lora_B, int r, float lora_scale, float* dA,
                                  float* dB, void* workspace, size_t workspace_bytes,
                                  e4b_stream stream);

/*
 * One grouped GEMM over E expert groups straight from MXFP4 expert bytes.
 * Source: Solutions -- one page per problem, the grouped-nf4-gemm row on
 * gemm_mxfp4_grouped (released e2m1 blocks and e8m0 scales multiplied as they
 * are, no requantisation, no bf16 weight copy).
 *
 * As e4b_grouped_nf4_gemm() (row p of group e: y[p, :] = A[row_index[p], :] .
 * W_e^T, the same epilogues, no adapter), with W_e in the OCP microscaling
 * format: element (n, k) = e2m1(code) * 2^(scale - 127), where
 *   blocks  [E, N*K/2] uint8: row n of expert e holds K/2 bytes, element 2i
 *           of the row in the low nibble of byte i (the released layout);
 *           e2m1 = sign (bit 3), exponent (bits 2-1, bias 1), mantissa (bit 0);
 *   scales  [E, N*K/32] uint8: one e8m0 byte per 32 consecutive elements of a
 *           row; 255 is NaN and makes its block NaN.
 * Requires K % 64 == 0, N % 64 == 0.
 * workspace  e4b_grouped_mxfp4_gemm_workspace_size() bytes: an error word and
 *            room for the routed rows gathered in order (total_rows x K bf16),
 *            which the tensor-core kernel (512 routed rows and more) reads as
 *            contiguous tiles; the warp-MMA kernel below uses neither.  0 bytes
 *            (NULL allowed) when total_rows == 0.
 * Each e2m1 value and each scale is exact in bf16, so the products with the
 * bf16 operand rows are the GEMM's only roundings (fp32 accumulation).
 */
E4B_API size_t e4b_grouped_mxfp4_gemm_workspace_size(int64_t total_rows, int64_t N, int64_t K);
E4B_API e4b_status e4b_grouped_mxfp4_gemm(const uint16_t* A, int64_t a_rows, int64_t lda,
                                  const int32_t* row_index, const int32_t* expert_offsets,
                                  int64_t E, int64_t total_rows, const uint8_t* blocks,
                                  const uint8_t* scales, int64_t N, int64_t K, e4b_epilogue epi,
                                  void* out, e4b_dtype out_dtype, void* workspace,
                                  size_t workspace_bytes, e4b_stream stream);

/* The two packed stacks of one MoE layer (device pointers), plus its adapter. */
typedef struct {
  const uint8_t* gu_packed; /* [E, 2I*H/2]  gate_up_proj, 4-bit codes */
  const float* gu_absmax;   /* [E, 2I*H/64] */
  const uint8_t* dn_packed; /* [E, H*I/2]   down_proj, 4-bit codes */
  const float* dn_absmax;   /* [E, H*I/64] */
  const uint16_t* lora_A;   /* [E, r, H] bf16 or NULL */
  const uint16_t* lora_B;   /* [E, 2I, r] bf16 or NULL */
  int lora_r;               /* 0 without an adapter */
  float lora_alpha;         /* scale = lora_alpha / lora_r */
  int64_t E, H, I;
  int32_t quant_type;       /* e4b_quant_type of both stacks; 0 (zero-initialised) = NF4 */
} e4b_expert_stack;

/*
 * a2..a8 -- the routed expert layer end to end:
 *     out[t] = sum_j w[t,j] * ( SiLU(g) * u ) . Wd_e^T,  [g | u] = x_t . Wgu_e^T (+ LoRA)
 * with (e, w[t,j]) from the top-k routing of router_logits[t].
 * Sources: as for the three calls above; the weighted sum over a token's
 * experts is the combine of experts4bit-qlora 0.22.0, "Which training path?".
 *
 * x [M, H] bf16, router_logits [M, E] fp32, out [M, H] bf16.
 * Requires H % 64 == 0, I % 64 == 0, 1 <= k <= min(E, 32), E <= 1024.
 * workspace  e4b_moe_expert_forward_workspace_size() bytes (covers both paths).
 * The sum over a token's k experts is taken in a fixed order for a given path,
 * so results are deterministic run to run.
 */
E4B_API size_t e4b_moe_expert_forward_workspace_size(int64_t M, const e4b_expert_stack* w, int k);
E4B_API e4b_status e4b_moe_expert_forward(const uint16_t* x, int64_t M, const float* router_logits,
                                  int k, int renormalize, const e4b_expert_stack* w,
                                  uint16_t* out, void* workspace, size_t workspace_bytes,
                                  e4b_stream stream);
/* Same, with the implementation chosen explicitly (tests and benchmarks).
 * E4B_PATH_AUTO takes the decode kernel when it can run the shape -- 1 <= M <= 8,
 * k <= 32, E <= 512, H <= 4096, I <= 3072 and its shared-memory plan fits -- and
 * the grouped path otherwise.  E4B_PATH_DECODE on any other shape returns
 * E4B_ERR_UNSUPPORTED and e4b_last_error() names the limit.
 * The decode path is one cooperative launch of one CTA per SM (at most 1024
 * CTAs): it needs the whole grid resident at once, so a launch that cannot get
 * every SM it asks for fails with E4B_ERR_CUDA instead of waiting.  Its CTAs
 * meet at a grid barrier whose slots and epoch word live in the workspace:
 * each call tags its slots with the epoch + 1 and advances the epoch, so a
 * workspace needs no initialisation for it (garbage, or the grouped path's
 * data, is fine) and graph replays work; two calls that share a workspace
 * must not overlap on the GPU. */
E4B_API e4b_status e4b_moe_expert_forward_path(const uint16_t* x, int64_t M, const float* router_logits,
                                       int k, int renormalize, const e4b_expert_stack* w,
                                       uint16_t* out, void* workspace, size_t workspace_bytes,
                                       e4b_path path, e4b_stream stream);

/*
 * Backward of the layer through the frozen NF4 experts, routing ids held fixed
 * (top-k selection is piecewise constant in the logits).
 * Source: experts4bit-qlora 0.22.0, "Which training path?" (per-expert LoRA
 * over a frozen NF4 stack; the base is decoded again in backward, one dgrad
 * launch per projection); Solutions -- one page per problem, the ExpertsLoRA row.
 *
 * For out = e4b_moe_expert_forward(x, router_logits, ...) and an upstream
 * gradient dout [M, H] bf16, writes the gradients of sum(dout * out):
 *   dx       [M, H] fp32    through gate_up and the adapter's delta
 *   dlogits  [M, E] fp32    through the routing weights (zero on unselected
 *                           experts with renormalisation)
 *   dA, dB   [E, r, H], [E, 2I, r] fp32, the adapter's gradients (required
 *            when the stack has an adapter, ignored otherwise)
 * The frozen stacks get no gradient.  It routes again, recomputes the gate_up
 * output (fp32) and the per-slot expert outputs (fp32), and runs the two
 * grouped dgrad products of e4b_grouped_nf4_gemm_dgrad() with the SwiGLU
 * derivative between them; every sum runs in a fixed order (deterministic).
 * workspace  e4b_moe_expert_backward_workspace_size() bytes (error word first).
 */
E4B_API size_t e4b_moe_expert_backward_workspace_size(int64_t M, const e4b_expert_stack* w, int k);
E4B_API e4b_status e4b_moe_expert_backward(const uint16_t* x, int64_t M, const float* router_logits,
                                   int k, int renormalize, const e4b_expert_stack* w,
                                   const uint16_t* dout, float* dx, float* dlogits, float* dA,
                                   float* dB, void* workspace, size_t workspace_bytes,
                                   e4b_stream stream);

/*
 * Allocation-free small-batch forward.  The pages have no counterpart of this
 * call; it exists for hosts that cannot give the library device memory:
 * serving engines that plan every byte of device memory into a fixed pool at
 * start-up, and runtimes that allow no allocator call (cudaMalloc or any
 * other) once their decode loop is running.
 *
 * Computes exactly what e4b_moe_expert_forward() computes for 1 <= M <= 8
 * tokens, with the decode kernel, but takes no workspace: its scratch (the
 * SwiGLU activations of the routed slots, M*k*I bf16 values, plus the slots
 * and epoch word of the kernel's grid barrier) lives in one statically
 * sized device array of the library, 528 KiB, which every GPU that loads the
 * library holds until the process exits.  Requires M*k*I <= 262144 (for example M = 8, k = 8,
 * I <= 4096); larger shapes return E4B_ERR_UNSUPPORTED with a message.  The
 * caller still owns x, router_logits, the stacks and out; nothing here calls
 * cudaMalloc, cudaFree or any allocating routine.
 *
 * The first call in each CUDA context looks up the device address of the
 * array (cudaGetSymbolAddress) with that context current, and caches it under
 * the context's unique id, so a context created after cudaDeviceReset gets a
 * fresh lookup.  With lazy module loading (CUDA_MODULE_LOADING=LAZY, the
 * default) the driver only materialises the library's module, and this
 * static array with it, at that first lookup or at the first launch of any
 * libe4b kernel: that is a device allocation made by the driver.  The promise
 * of no allocation therefore holds from the second call on: make one eager
 * call on each device (or context) during start-up, before any stream capture
 * and outside the decode loop.  All calls share the one array and it keeps
 * the last call's contents, so calls whose kernels overlap on the GPU
 * (different streams without ordering between them) race and give wrong
 * results.
 */
E4B_API e4b_status e4b_moe_expert_forward_decode_noalloc(const uint16_t* x, int64_t M,
                                                         const float* router_logits, int k,
                                                         int renormalize, const e4b_expert_stack* w,
                                                         uint16_t* out, e4b_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* E4B_H_ */

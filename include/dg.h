/*
 * dg.h — C ABI of the B200 (sm_100a) FP8 block-scaled GEMM library (libdg.so).
 *
 * Operation (DeepGEMM pages: "DeepGEMM 简介" and "4 DeepGEMM 架构分析 — 两级累加结构"
 * on the juejin.cn Open-Source-Week article; "Per-block scaling 通过 CUDA-core
 * promotion" and "UE8M0 int32 packing" on the nightvoyager.top GitHub report):
 *
 *   D[m,n] = bf16_rne( sum_kb sa[m,kb] * sb[n/128,kb]
 *                             * sum_{k in 128-wide block kb} A[m,k] * B[n,k] )
 *
 * A, B are FP8 E4M3; sa is one power-of-two scale per row of A and 128-wide K
 * block (1x128), sb one per 128x128 block of B; both are UE8M0 exponents
 * packed four per int32.  D is BF16, overwritten (no C input).
 *
 * Conventions shared by every entry point
 *  - Every data pointer is DEVICE memory owned by the caller, 16-byte aligned.
 *    The library allocates nothing per call; it keeps only a per-device
 *    error word.  `stream` is a cudaStream_t (NULL = legacy default stream);
 *    calls are asynchronous and stream-ordered.
 *  - Layouts are row-major and dense.  "NT": A is [M,K] and B is [N,K], both
 *    K-contiguous; D is [M,N], N-contiguous.
 *  - Packed scales ("TMA-aligned, transposed" layout of the ssnai.com DeepGEMM
 *    analysis, FP8 pitfalls block): a matrix of scales with MN rows and Kb = K/128
 *    blocks is stored as int32 words [ceil(Kb/4)][align4(MN)], MN contiguous;
 *    byte j (bits 8j..8j+7) of word [kp][mn] is the UE8M0 exponent e of block
 *    4*kp+j, meaning 2^(e-127).  Padding bytes are 0.  For A, MN = rows of A;
 *    for B, MN = ceil(N/128).
 *  - Requirements: K % 128 == 0 and K > 0; N % 16 == 0 and N > 0; M >= 0.
 *  - Return value: DG_OK or a negative dg_status.  Argument errors are found on
 *    the host before anything is launched (the C counterpart of DeepGEMM's
 *    host asserts); dg_get_last_error() then describes the problem.
 *    Data-dependent errors (expert index out of range, masked_m outside
 *    [0, M_max], a scale that is not a power of two) are found on the device:
 *    the kernel skips or clamps the offending item, sets a bit in the device
 *    error word and returns normally.  Read it with dg_get_device_error().
 */
#ifndef DG_H_
#define DG_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DG_OK = 0,
  DG_ERR_NULL = -1,        /* a required pointer is NULL                     */
  DG_ERR_SHAPE = -2,       /* a size violates the requirements above         */
  DG_ERR_ALIGN = -3,       /* a pointer is not 16-byte aligned               */
  DG_ERR_UNSUPPORTED = -4, /* no GPU / not sm_100 / configuration not built  */
  DG_ERR_CUDA = -5,        /* a CUDA runtime or driver call failed           */
  DG_ERR_DEVICE_DATA = -6, /* reported by dg_get_device_error                */
  DG_ERR_TIMEOUT = -7      /* reported by dg_get_device_error                */
} dg_status;

/* Bits of the device error word. */
#define DG_DEVERR_BAD_SCALE     0x1  /* pack: a scale is not a power of two in UE8M0 range */
#define DG_DEVERR_BAD_EXPERT    0x2  /* contiguous: m_indices value < -1 or >= num_groups  */
#define DG_DEVERR_BAD_MASKED_M  0x4  /* masked: masked_m[g] < 0 or > M_max (clamped)       */
#define DG_DEVERR_MIXED_TILE    0x8  /* contiguous: a 128-row tile holds two experts       */
#define DG_DEVERR_TIMEOUT       0x10 /* a pipeline wait exceeded its time limit; CTA quit   */

/*
 * Dense FP8 GEMM, NT layout (juejin.cn article §5 "常规稠密 GEMM"; the
 * nightvoyager.top report's "fp8_gemm_nt(a, b, d, c=None, ...)" signature).
 *   a   : E4M3 [M][K]                 sfa : packed scales, MN = M
 *   b   : E4M3 [N][K]                 sfb : packed scales, MN = ceil(N/128)
 *   d   : BF16 [M][N], written in full (M == 0 is a no-op).
 */
int dg_fp8_gemm_nt(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb, void* d,
                   int M, int N, int K, void* stream);

/*
 * The three GEMMs of the hot path with A's scales given as fp32 powers of two
 * instead of packed words: sfa is float [M][K/128] (dense), [M_total][K/128]
 * (contiguous) or [G][M_max][K/128] (masked), row-major, 4-byte aligned.  The
 * kernel's scale-producer warp packs each group of four exponents as
 * dg_pack_sf_ue8m0 would (the nightvoyager.top report, "SF 双 path": the
 * library turns FP32 scales into the packed UE8M0 layout), so a step needs
 * no separate packing launch.  A scale that is not a power of two in UE8M0
 * range is used as 2^-127 and sets DG_DEVERR_BAD_SCALE.  Everything else
 * (B's packed scales, layouts, errors) is as in the packed-word entry points.
 */
int dg_fp8_gemm_nt_fp32sfa(const void* a, const float* sfa, const void* b, const int32_t* sfb, void* d,
                           int M, int N, int K, void* stream);
int dg_m_grouped_fp8_gemm_nt_contiguous_fp32sfa(const void* a, const float* sfa, const void* b,
                                                const int32_t* sfb, void* d, const int32_t* m_indices,
                                                int M_total, int N, int K, int num_groups, void* stream);
int dg_m_grouped_fp8_gemm_nt_masked_fp32sfa(const void* a, const float* sfa, const void* b,
                                            const int32_t* sfb, void* d, const int32_t* masked_m,
                                            int num_groups, int M_max, int N, int K, void* stream);

/*
 * Dense FP8 GEMM with the other operand layouts (the ssnai.com analysis,
 * "SM90 vs SM100": SM100 serves NT, TN, NN and TT).  The first letter is the
 * LHS, the second the RHS; N = not transposed, T = transposed, so NT is
 * A [M][K] with B [N][K].  The product and the scales are those of
 * dg_fp8_gemm_nt: D[m][n] = sum_k A(m,k) B(n,k) with A's 1x128 scales along
 * K per row m and B's 128x128 block scales (same packed layouts).  Only the
 * storage of the FP8 operands changes:
 *   NN : a = A  as [M][K] (K contiguous),  b = B  as [K][N] (N contiguous)
 *   TN : a = A  as [K][M] (M contiguous),  b = B  as [K][N] (N contiguous)
 *   TT : a = A  as [K][M] (M contiguous),  b = B  as [N][K] (K contiguous)
 * The tensor core reads the M- or N-contiguous tiles directly; nothing is
 * transposed in memory.  Extra requirement: M % 16 == 0 when a is [K][M]
 * (16-byte row stride).  Tiles: B stored [K][N] uses 128- or 256-wide N
 * tiles.  Errors and ownership as dg_fp8_gemm_nt.
 */
int dg_fp8_gemm_nn(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb, void* d,
                   int M, int N, int K, void* stream);
int dg_fp8_gemm_tn(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb, void* d,
                   int M, int N, int K, void* stream);
int dg_fp8_gemm_tt(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb, void* d,
                   int M, int N, int K, void* stream);

/*
 * Dense FP8 GEMM, NT layout, with the recipe and output options of DeepGEMM's
 * `fp8_gemm_nt(a, b, d, c=None, recipe=...)` (nightvoyager.top report, "解法哲学";
 * "1d1d / 1d2d" kernels under "关键设计决策"; the juejin.cn article §2.1's
 * general GEMM C = alpha*A*B + beta*C with alpha = beta = 1):
 *   sfb_gran_n : 128 -> B scales per 128x128 block (packed MN = ceil(N/128));
 *                1   -> B scales per row and 128-wide K block, "1D1D" (packed MN = N).
 *   c          : optional FP32 [M][N] added to the product (NULL: none); needs d_is_fp32.
 *   d          : BF16 [M][N] (d_is_fp32 = 0) or FP32 [M][N] (d_is_fp32 = 1).
 * With c == NULL, sfb_gran_n == 128 and d_is_fp32 == 0 this is dg_fp8_gemm_nt.
 */
int dg_fp8_gemm_nt_ex(const void* a, const int32_t* sfa, const void* b, const int32_t* sfb, const float* c,
                      void* d, int M, int N, int K, int sfb_gran_n, int d_is_fp32, void* stream);

/*
 * M-grouped GEMM, contiguous layout (juejin.cn article §4 "分组 GEMM（连续布局）":
 * the experts' tokens are concatenated along M, each expert segment aligned
 * to the M block; N and K are shared by all experts).
 *   a         : E4M3 [M_total][K]     sfa : packed scales, MN = M_total
 *   b         : E4M3 [G][N][K]        sfb : G packed matrices, MN = ceil(N/128)
 *   d         : BF16 [M_total][N]
 *   m_indices : int32 [M_total], expert of each row, -1 for padding rows.
 * M_total must be a multiple of 128 (dg_get_mk_alignment_for_contiguous_layout)
 * and every aligned 128-row tile must hold rows of one expert (plus -1 rows).
 * Rows with index -1 are not written.  A tile whose first row is -1 is
 * skipped entirely.  Out-of-range indices set DG_DEVERR_BAD_EXPERT and their
 * rows are not written; rows of a second expert inside a tile set
 * DG_DEVERR_MIXED_TILE and are not written.
 */
int dg_m_grouped_fp8_gemm_nt_contiguous(const void* a, const int32_t* sfa, const void* b,
                                        const int32_t* sfb, void* d, const int32_t* m_indices,
                                        int M_total, int N, int K, int num_groups, void* stream);

/*
 * M-grouped GEMM, masked layout (juejin.cn article §4 "分组 GEMM（掩码分组）":
 * fixed per-expert capacity plus a device-side valid count, so the call can be
 * captured in a CUDA graph while token counts change).
 *   a        : E4M3 [G][M_max][K]     sfa : G packed matrices, MN = M_max
 *   b        : E4M3 [G][N][K]         sfb : G packed matrices, MN = ceil(N/128)
 *   d        : BF16 [G][M_max][N]
 *   masked_m : int32 [G] on the device, valid rows of each expert; read by the
 *              kernel, never by the host.  Rows m >= masked_m[g] of expert g
 *              are not written.  Values outside [0, M_max] are clamped and set
 *              DG_DEVERR_BAD_MASKED_M.
 */
int dg_m_grouped_fp8_gemm_nt_masked(const void* a, const int32_t* sfa, const void* b,
                                    const int32_t* sfb, void* d, const int32_t* masked_m,
                                    int num_groups, int M_max, int N, int K, void* stream);

/*
 * Packs fp32 power-of-two scales into the UE8M0 int32 layout above
 * (nightvoyager.top report, "SF 双 path 缓存设计": float32 scales go through a
 * transform kernel once, e.g. for weights, and the packed words are reused).
 *   sf     : fp32 [batch][mn][kb]          (device)
 *   packed : int32 [batch][ceil(kb/4)][align4(mn)]   (device, fully written)
 * A valid scale is a positive normal fp32 power of two, or 2^-127 (byte 0).
 * Anything else writes byte 0 and sets DG_DEVERR_BAD_SCALE.
 */
int dg_pack_sf_ue8m0(const float* sf, int32_t* packed, int batch, int mn, int kb, void* stream);

/*
 * Per-token FP8 quantisation of activations, fused with the scale packing:
 * the step before the GEMM that DeepGEMM leaves to its caller (ssnai.com
 * analysis, "库不做预处理" / "上层完成转置与 FP8/FP4 casting").
 *   x       : [batch][M][K] activations, BF16 (x_dtype 0) or FP32 (x_dtype 1), finite
 *   q       : E4M3 [batch][M][K] (written)
 *   sf      : int32 [batch][ceil(K/512)][align4(M)] packed UE8M0 scales (written,
 *             padding included): the `sfa` layout of the GEMM entry points.
 * For every row and 128-wide K group the scale is the smallest power of two s
 * with max|x|/s <= 448 (1 for an all-zero group, clamped to [2^-127, 2^127])
 * and q = E4M3(x/s), round to nearest even, saturating.  K % 128 == 0.
 */
int dg_quantize_fp8_1x128(const void* x, int x_dtype, void* q, int32_t* sf, int batch, int M, int K,
                          void* stream);

/*
 * MoE permutation into the contiguous layout ("group_by_expert", the step
 * before the grouped GEMM in the charles2530.github.io source guide §七) and
 * the weighted combine after it.
 *
 * dg_moe_permute_capacity: rows that always suffice for M_cap,
 *   align128(T*topk + 127*num_experts).
 * dg_moe_permute:
 *   topk_ids : int32 [T][topk], expert of each routed slot, -1 = not routed
 *   q, sfa   : the tokens' E4M3 codes [T][K] and packed scales [ceil(K/512)][align4(T)]
 *              (as written by dg_quantize_fp8_1x128)
 *   a_perm   : E4M3 [M_cap][K]   sfa_perm : int32 [ceil(K/512)][M_cap]
 *   m_indices: int32 [M_cap]     src_of   : int32 [M_cap] source token of each row (-1: padding)
 *   row_of   : int32 [T][topk], row of each routed slot (-1: not routed)
 * Expert segments follow in expert order, each padded with -1 rows to a multiple
 * of 128; inside a segment slots keep their (token, slot) order, so the result is
 * deterministic.  Rows past the last segment are -1.  a_perm / sfa_perm / m_indices
 * feed dg_m_grouped_fp8_gemm_nt_contiguous with M_total = M_cap directly.
 * The codes of padding and tail rows of a_perm are not written (their scale words
 * are written as 0, and the grouped GEMM never stores those rows).
 * Ids outside [-1, num_experts) set DG_DEVERR_BAD_EXPERT and are not routed.
 * num_experts <= 1024; M_cap >= dg_moe_permute_capacity(...) and a multiple of 128.
 * With T = 0, topk_ids, q, sfa and row_of may be NULL: every row becomes padding.
 * dg_moe_unpermute_combine:
 *   out[t] = bf16_rne( sum_s weights[t][s] * d_perm[row_of[t][s]] ) in FP32 over routed
 *   slots (weights NULL = 1); d_perm BF16 [rows][N], out BF16 [T][N], N % 16 == 0.
 *   Every row_of entry must be -1 or a row of d_perm.  The call has no row count of
 *   d_perm to check them against (row_of is device data), so this is the caller's
 *   contract; row_of from dg_moe_permute with d_perm of M_cap rows meets it.
 */
int dg_moe_permute_capacity(int T, int topk, int num_experts);
int dg_moe_permute(const int32_t* topk_ids, int T, int topk, int num_experts, const void* q, const int32_t* sfa, int K,
                   void* a_perm, int32_t* sfa_perm, int32_t* m_indices, int32_t* row_of, int32_t* src_of, int M_cap,
                   void* stream);
int dg_moe_unpermute_combine(const void* d_perm, const int32_t* row_of, const float* weights, int T, int topk, int N,
                             void* out, void* stream);

/* M alignment of expert segments in the contiguous layout (128). */
int dg_get_mk_alignment_for_contiguous_layout(void);

/* Number of int32 words of one packed scale matrix: ceil(kb/4) * align4(mn). */
int64_t dg_packed_sf_words(int mn, int kb);

/* Returns the current device's error word in *err (0 = none, else DG_DEVERR_*
 * bits) and clears it, in one atomic step on the device that is ordered after
 * the earlier work of `stream`; then synchronises `stream`.  Bits that
 * kernels on other streams set meanwhile stay in the word for the next read.
 * (Failure contract of the nightvoyager.top report's "解法哲学": errors are
 * reported, not trapped.) */
int dg_get_device_error(void* stream, int* err);

/* Time limit of each pipeline wait inside the GEMM kernels, in nanoseconds,
 * for every later call in this process (default 2e9, i.e. 2 s).  A wait that
 * runs out sets DG_DEVERR_TIMEOUT; every role of that CTA then stops
 * issuing, waits (with the 2 s limit, whatever this setting) for its own
 * copies and tensor-core operations in flight, frees its tensor memory and
 * exits, so the context stays usable and the output is incomplete.  A short
 * limit (0 included) makes an ordinary call give up: it exists to exercise
 * that path.  Returns the previous limit. */
uint64_t dg_set_wait_limit_ns(uint64_t ns);

/* Persistent-grid size (the ssnai.com analysis' set_num_sms knob).
 * n <= 0 restores "all SMs".  Returns the previous setting. */
int dg_set_num_sms(int n);
int dg_get_num_sms(void);

/* Share of the GPU's tensor cores a call may occupy, in percent (1..100,
 * 100 = all; the ssnai.com analysis lists set_tc_util beside set_num_sms
 * and set_pdl as run-time tuning knobs, e.g. to leave SMs to a concurrent
 * communication kernel).  Read here as a cap on the SMs a call plans and
 * launches for: floor(SMs x percent / 100), at least one CTA pair, after
 * dg_set_num_sms.  Returns the previous setting, or DG_ERR_SHAPE. */
int dg_set_tc_util(int percent);

/* Programmatic dependent launch for every kernel of this library (on by
 * default): a kernel's set-up (barrier init, tensor-memory allocation) may
 * overlap the end of the previous kernel on the stream; the kernel waits for
 * that kernel's completion before its first global-memory access, so stream
 * order is kept.  enable = 0 launches plainly.  Returns the previous setting. */
int dg_set_pdl(int enable);

/* The three knobs above take their initial values from the environment when
 * the library is loaded: DG_NUM_SMS (integer >= 0), DG_TC_UTIL (1..100) and
 * DG_PDL (0 or 1).  Unset or malformed variables leave the defaults (all SMs,
 * 100 %, PDL on).  The setters override them at any time. */

/* Forces the tile configuration of the next calls on this host thread:
 * block_n (an N tile width), ctas (1: 128-row tiles on one SM; 2: 256-row
 * tiles on a pair of SMs; 0: the first built) and pipes (1: one load/MMA
 * pipeline per CTA; 2: two pipelines, each with its own MMA-issuing thread
 * and accumulator; 0: the first built).  block_n == 0 restores the heuristic.
 * Built (block_n, ctas, pipes) triples:
 *   dense NT and masked : (64|128|224|256, 1, 1), (128|224|256, 2, 1),
 *                         (128|224, 2, 2) alternate tiles over the pipelines,
 *                         (64|128, 1, 2) split-K: both pipelines on every tile,
 *                         each over half of K (used for problems of <= 128 rows)
 *   contiguous          : (128|224|256, 1, 1), (224, 2, 2)
 *   FP32 output (_ex)   : (128|224|256, 1, 1)
 *   NN / TN / TT        : fewer tiles.
 * The triple must be built for at least one entry point (else
 * DG_ERR_UNSUPPORTED).  An entry point that does not build it keeps the
 * heuristic's choice. */
int dg_set_config(int block_n, int ctas, int pipes);

/* Describes the configuration the heuristic picks for a problem, as
 * "BMxBNxSTAGES[(2cta)]/grid" in buf (kind: 0 dense, 1 contiguous, 2 masked). */
int dg_describe_config(int kind, int M, int N, int K, int num_groups, char* buf, int buflen);

/* Text of the last host-side error on this thread ("" if none). */
const char* dg_get_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* DG_H_ */

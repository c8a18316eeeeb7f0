/*
 * dg.h -- C ABI of the B200 (sm_100a) FP8 block-scaled NT GEMM library.
 *
 * Operation (page "DeepGEMM项目介绍与本地部署指南" -- DeepGEMM project
 * introduction and local deployment guide -- section "接口" (Interface); scale
 * granularity and the 128-wide promotion interval from the page "Deepseek
 * DeepGEMM 技术原理的深入分析", section "技术背景与核心原理"):
 *
 *   D[m,n] = bf16( sum_kb sa[m,kb] * sb[n/128,kb] * sum_{k in block kb} A[m,k]*B[n,k] )
 *
 * with A, B in FP8 e4m3 (OCP E4M3FN), FP32 scales per 1x128 row tile of A (sa)
 * and per 128x128 block of B (sb), FP32 accumulation in which every 128-wide
 * K block's partial product is scaled and added separately, and a bf16 result
 * rounded to nearest even.
 *
 * Common conventions for every entry point below
 * ----------------------------------------------
 *  Pointers   All tensor pointers are CUDA DEVICE pointers, 16-byte aligned,
 *             owned by the caller.  The library never allocates, frees or
 *             keeps them past the call.
 *  Workspace  Dense calls whose last wave of tiles is partial split those
 *             tiles along K; the slices' FP32 partials go to a workspace the
 *             library allocates once per (device, stream) on first need (one
 *             128 x BN FP32 tile per SM, about 19 MB on a B200, zeroed).  At
 *             most four streams per device hold one: the first split call on
 *             a fifth stream frees the least recently used workspace (its
 *             cudaFree waits for the device), so short-lived streams do not
 *             accumulate memory.  While a stream is being captured into a CUDA
 *             graph and has no workspace yet, calls do not split (results are
 *             the same up to FP32 summation order); make one call on the
 *             stream before capturing to keep the split, and capture on at
 *             most four streams per device that way.  dg_get_device_error()
 *             clears the workspaces' ready flags when it reports
 *             DG_DEVERR_TIMEOUT, so a timed-out launch leaves none set.
 *  Layouts    A   uint8 (e4m3 codes) [rows][K], K contiguous.
 *             B   uint8 (e4m3 codes) [G][N][K], K contiguous ("NT": the RHS is
 *                 stored transposed).  G = 1 for the dense call.
 *             sa  float32, TRANSPOSED: element (m, kb) at sa[kb*sa_stride + m]
 *                 (masked: group g's block starts at g*ceil(K/128)*sa_stride).
 *                 sa_stride >= rows and a multiple of 4 (16 bytes), e.g.
 *                 dg_get_tma_aligned_size(rows, 4).
 *             sb  float32 [G][ceil(N/128)][ceil(K/128)], row-major.
 *             D   bf16 bits (uint16) [rows][N] row-major (masked: [G][M_max][N]).
 *  Limits     K % 128 == 0, N % 8 == 0 (16-byte rows of D), K and N >= 1.
 *  Stream     `stream` is a cudaStream_t (NULL = legacy default stream).  The
 *             call only enqueues work: it does not synchronise, read device
 *             memory from the host, or allocate, so it may be captured in a
 *             CUDA graph.
 *  Errors     Bad arguments are reported synchronously as a dg_status and
 *             nothing is launched (dg_last_error_message() says why).  A
 *             launch failure returns DG_ERR_CUDA.  DG_ERR_UNSUPPORTED also
 *             reports a library build whose kernel cannot run as compiled:
 *             before a kernel's first launch the host checks that its
 *             compiled register count covers the kernel's register split
 *             (threads x registers per thread), which would otherwise wait
 *             forever on the device.  Bad DEVICE-side data
 *             (m_indices outside [-1,G), masked_m outside [0,M_max]) cannot be
 *             seen by the host: the kernel skips the offending rows/groups
 *             (masked_m is clamped) and sets a bit in the device error word,
 *             read with dg_get_device_error().  Every wait inside the kernels
 *             is bounded; a wait that runs out sets DG_DEVERR_TIMEOUT and the
 *             kernel returns instead of hanging.
 *  Threads    dg_set_num_sms() is process-global; all other calls are
 *             reentrant.
 */
#ifndef DG_H_
#define DG_H_

#include <stdint.h>

#if defined(__GNUC__)
#define DG_API __attribute__((visibility("default")))
#else
#define DG_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum dg_status {
    DG_OK = 0,
    DG_ERR_INVALID_ARG = 1,  /* null pointer, non-positive size, bad stride     */
    DG_ERR_UNSUPPORTED = 2,  /* valid in the math but not on this path (K%128)  */
    DG_ERR_MISALIGNED = 3,   /* a pointer is not 16-byte aligned                */
    DG_ERR_CUDA = 4          /* a CUDA runtime/driver call or launch failed     */
} dg_status;

/* Bits of the device error word (dg_get_device_error). */
#define DG_DEVERR_TIMEOUT 1u        /* a bounded wait inside a kernel ran out  */
#define DG_DEVERR_BAD_M_INDEX 2u    /* contiguous: m_indices value not in [-1,G) */
#define DG_DEVERR_BAD_MASKED_M 4u   /* masked: masked_m value not in [0,M_max]  */
#define DG_DEVERR_NOT_POW2 8u       /* ue8m0 call: a scale is not a positive     */
                                    /* normal power of two                       */
#define DG_DEVERR_BAD_K_OFFSET 16u  /* K-grouped: k_offsets not increasing       */
                                    /* multiples of 128 within [0, K]            */

/*
 * Dense GEMM: D[M,N] = scaled A[M,K] . B[N,K]^T (section "常规密集型 GEMM（非分组）",
 * the non-grouped call of the Interface section).
 *   D          uint16 bf16 [M][N]
 *   A          uint8 e4m3 [M][K]
 *   sa         float32 transposed, sa[kb*sa_stride + m], kb < K/128
 *   B          uint8 e4m3 [N][K]
 *   sb         float32 [ceil(N/128)][K/128]
 * M == 0 is a valid empty problem (returns DG_OK, launches nothing).
 */
DG_API dg_status dg_fp8_gemm_nt(uint16_t* D, const uint8_t* A, const float* sa, int sa_stride,
                         const uint8_t* B, const float* sb, int M, int N, int K, void* stream);

/*
 * Dense GEMM with the operands in the other storage orders.  The later-version
 * article on DeepGEMM (section 3.1) notes that from SM100 on all four layouts
 * NT, TN, NN and TT are supported.  The product is the same D = A . B^T with
 * logical A [M][K] and B [N][K] and the same scales (sa transposed per 1x128,
 * sb [ceil(N/128)][K/128]); only where A and B live changes:
 *   dg_fp8_gemm_nn   A [M][K] (K contiguous),   B stored [K][N] (N contiguous)
 *   dg_fp8_gemm_tn   A stored [K][M] (M contiguous), B stored [K][N]
 *   dg_fp8_gemm_tt   A stored [K][M],           B [N][K] (K contiguous)
 * (dg_fp8_gemm_nt is A [M][K], B [N][K].)  A stored [K][M] needs M % 16 == 0,
 * B stored [K][N] needs N % 16 == 0 (16-byte rows for TMA); otherwise the
 * limits of dg_fp8_gemm_nt hold.  These calls always use the 128 x {128,256}
 * tile kernel (no few-row kernel).
 */
DG_API dg_status dg_fp8_gemm_nn(uint16_t* D, const uint8_t* A, const float* sa, int sa_stride,
                                const uint8_t* B, const float* sb, int M, int N, int K, void* stream);
DG_API dg_status dg_fp8_gemm_tn(uint16_t* D, const uint8_t* A, const float* sa, int sa_stride,
                                const uint8_t* B, const float* sb, int M, int N, int K, void* stream);
DG_API dg_status dg_fp8_gemm_tt(uint16_t* D, const uint8_t* A, const float* sa, int sa_stride,
                                const uint8_t* B, const float* sb, int M, int N, int K, void* stream);

/*
 * Grouped GEMM along K (the weight-gradient GEMM of a MoE layer; the
 * later-version article on DeepGEMM, section 3.2, names grouping along M or
 * along K).  Group g owns the K rows [k_offsets[g], k_offsets[g+1]) -- e.g.
 * the tokens routed to expert g -- and
 *   D[g][m][n] = bf16( sum over g's K blocks kb of sa[m,kb]*sb[n/128,kb]*P_kb[m,n] ),
 * the dense formula restricted to the group's K blocks (an empty group gives
 * zeros).  Storage as in dg_fp8_gemm_tn, with K the total over all groups:
 *   A          uint8 e4m3 stored [K][M] (M contiguous, M % 16 == 0)
 *   B          uint8 e4m3 stored [K][N] (N contiguous, N % 16 == 0)
 *   sa         float32, sa[kb*sa_stride + m], kb < K/128 (global K blocks)
 *   sb         float32 [ceil(N/128)][K/128]
 *   k_offsets  int32 [G+1] on the device, increasing multiples of 128 with
 *              k_offsets[G] <= K; bad values set DG_DEVERR_BAD_K_OFFSET and the
 *              group's D is written as zeros
 *   D          bf16 [G][M][N]
 * M == 0 is valid and launches nothing.
 */
DG_API dg_status dg_k_grouped_fp8_gemm_tn(uint16_t* D, const uint8_t* A, const float* sa, int sa_stride,
                                          const uint8_t* B, const float* sb, const int32_t* k_offsets, int G,
                                          int M, int N, int K, void* stream);

/*
 * Dense GEMM for power-of-two scales, scaled inside the tensor core.  Same
 * arguments, layouts and result as dg_fp8_gemm_nt, but every sa and sb value
 * must be a positive normal power of two (UE8M0-representable: its FP32
 * exponent field is the UE8M0 code).  The later-version article on DeepGEMM
 * (section 3.1) notes that SM100 takes UE8M0 scales; this call hands them to
 * tcgen05.mma kind::mxf8f6f4.block_scale, which applies them to each K=32
 * partial product before the FP32 accumulation, instead of promoting every
 * 128-K block through registers.  The result is the method's sum up to FP32
 * summation order (tolerance as for dg_fp8_gemm_nt).  A scale that is not a
 * power of two sets DG_DEVERR_NOT_POW2 in the device error word and its tile's
 * results are then wrong; the call does not check the scales on the host.
 * The block-scaled kernel is used for M > 256, where it measured faster than
 * the promotion kernel; fewer rows take the promotion path (the same result,
 * no DG_DEVERR_NOT_POW2 check).  DG_FORCE_BLOCK_SCALED=1 in the environment
 * forces the block-scaled kernel, =0 the promotion path.  Like
 * dg_fp8_gemm_nt, the call may split the tiles of a partial last wave (or all
 * tiles, when there are fewer than SMs) along K; the split uses the stream's
 * K-split workspace (see "Workspace" above) and is deterministic.
 */
DG_API dg_status dg_fp8_gemm_nt_ue8m0(uint16_t* D, const uint8_t* A, const float* sa, int sa_stride,
                                      const uint8_t* B, const float* sb, int M, int N, int K, void* stream);

/*
 * Number of K-split workspaces (see "Workspace" above) the library holds,
 * over all devices and streams.  Host-only, no synchronisation; for tests and
 * memory accounting.
 */
DG_API int dg_get_workspace_count(void);

/*
 * Dense GEMM that allocates nothing.  The pages describe no such call; it
 * exists for callers that must not allocate device memory once they are
 * running: a serving loop that reserved all of HBM for its own pool up front,
 * or code that cannot afford the device-wide synchronisation cudaMalloc and
 * cudaFree may bring.  Same arguments, layouts and result as dg_fp8_gemm_nt.
 *
 * Where the last wave of tiles is split along K, its FP32 partials and flags
 * live in one static device array of 16 MiB + 4 KiB, held on every GPU that
 * loads the library until the process exits, instead of in a workspace the
 * library allocates.  A call whose split would need more than that returns
 * DG_ERR_UNSUPPORTED and launches nothing (on a 148-SM B200 no call does).
 * The flags are cleared on the stream before each launch that uses them.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture starts.
 *   - Every call on a device shares the one array: calls that may overlap on
 *     the GPU (other streams, or a concurrent thread) race on it and give
 *     wrong results.  Order them on one stream or with events.
 */
DG_API dg_status dg_fp8_gemm_nt_noalloc(uint16_t* D, const uint8_t* A, const float* sa, int sa_stride,
                                        const uint8_t* B, const float* sb, int M, int N, int K, void* stream);

/*
 * FP8 cast of activations (the GEMM's A and sa).  The pages leave the cast to
 * the caller ("接口": e4m3 inputs, transposed TMA-aligned LHS scales) and name
 * a helper to_fp8 returning the FP8 tensor with its scale factors (the
 * later-version article on DeepGEMM, section 4.1); one scale per 1x128 tile
 * ("Deepseek DeepGEMM 技术原理的深入分析", section "技术背景与核心原理").
 * Per tile, in IEEE single precision:
 *   amax = max(max |x|, 1e-4),  s = amax / 448,
 *   q = e4m3 of x * (448 / amax), round to nearest even, saturating to +-448
 *   (NaN in, NaN out).
 *   Q          uint8 e4m3 [M][K] (written)
 *   sa         float32, sa[kb*sa_stride + m], kb < K/128 (written; the rest of
 *              each sa_stride run is left untouched)
 *   X          uint16 bf16 [M][K] (read)
 * K % 128 == 0, sa_stride >= M (a multiple of 4 for the GEMM's TMA), X and Q
 * 16-byte aligned.  M == 0 is valid and launches nothing.
 */
DG_API dg_status dg_to_fp8_1x128(uint8_t* Q, float* sa, int sa_stride, const uint16_t* X, int M, int K,
                                 void* stream);

/*
 * FP8 cast of weights (the GEMM's B and sb), one scale per 128x128 block, the
 * same steps as dg_to_fp8_1x128 over each block (the last row block may be
 * shorter than 128).
 *   Q          uint8 e4m3 [N][K] (written)
 *   sb         float32 [ceil(N/128)][K/128], row-major (written)
 *   W          uint16 bf16 [N][K] (read)
 * K % 128 == 0, W and Q 16-byte aligned.  N == 0 is valid and launches nothing.
 * For a grouped [G][N][K] weight, call once per group with the group's slices.
 */
DG_API dg_status dg_to_fp8_128x128(uint8_t* Q, float* sb, const uint16_t* W, int N, int K, void* stream);

/*
 * Grouped GEMM, contiguous layout (section "分组 GEMM（连续布局）"): the rows of
 * all groups are concatenated along M and share N and K.  m_indices[m] (int32,
 * device) is the group of row m; -1 marks a padding row, whose D row is left
 * untouched.  Each group's segment must start on a multiple of
 * dg_get_m_alignment_for_contiguous_layout() rows, so M_total is a multiple
 * of it.  Row m uses B + g*N*K and sb + g*ceil(N/128)*(K/128).
 *   D [M_total][N], A [M_total][K], sa transposed with sa_stride >= M_total,
 *   B [G][N][K], sb [G][ceil(N/128)][K/128], m_indices [M_total].
 */
DG_API dg_status dg_grouped_contiguous_nt(uint16_t* D, const uint8_t* A, const float* sa, int sa_stride,
                                   const uint8_t* B, const float* sb, const int32_t* m_indices,
                                   int M_total, int N, int K, int G, void* stream);

/*
 * Grouped GEMM, masked layout (section "分组 GEMM（掩码布局）"): for decoding
 * under CUDA graphs, where the host does not know how many rows each group
 * holds.  masked_m[g] (int32, device) rows of group g are computed; rows
 * masked_m[g] .. M_max-1 of D[g] are left untouched.  The launch does not
 * depend on masked_m.
 *   D [G][M_max][N], A [G][M_max][K],
 *   sa [G][K/128][sa_stride] (transposed per group, sa_stride >= M_max),
 *   B [G][N][K], sb [G][ceil(N/128)][K/128], masked_m [G].
 *   expected_m  host hint of the typical masked_m (<= 0: unknown); it may
 *               change the tile shape chosen, never the result.
 */
DG_API dg_status dg_grouped_masked_nt(uint16_t* D, const uint8_t* A, const float* sa, int sa_stride,
                               const uint8_t* B, const float* sb, const int32_t* masked_m,
                               int G, int M_max, int N, int K, int expected_m, void* stream);

/* Utility functions (section "工具函数" (utility functions) of the same page). */

/*
 * Programmatic dependent launch (the later-version article on DeepGEMM,
 * section 4.3, enables it with set_pdl(True)).  When on, every launch of this
 * library may start its set-up while the previous kernel in the stream is
 * finishing; the kernels wait for that kernel's results before touching global
 * memory, so results never change.  On by default (measured: about 1 us less
 * per decode-sized launch in back-to-back CUDA-graph replays).
 *   dg_set_pdl(1) on, dg_set_pdl(0) off, dg_set_pdl(-1) back to the default,
 *   which is on unless the environment variable DG_PDL=0 at the launch.
 * Process-global, like dg_set_num_sms.  dg_get_pdl returns the current state.
 */
DG_API void dg_set_pdl(int enable);
DG_API int dg_get_pdl(void);

/* Cap the number of SMs the persistent kernels use (n <= 0: all SMs). */
DG_API void dg_set_num_sms(int n);
/* Current cap; the device's SM count when no cap is set (0 without a GPU). */
DG_API int dg_get_num_sms(void);
/* Row alignment every group segment needs in the contiguous layout (128). */
DG_API int dg_get_m_alignment_for_contiguous_layout(void);
/* x rounded up so that x*elem_bytes is a multiple of 16 bytes (TMA stride rule). */
DG_API int dg_get_tma_aligned_size(int x, int elem_bytes);

/* Reads the device error word of the current device, clears it, and stores it
 * in *code.  Synchronises the device first; meant for tests and debugging. */
DG_API dg_status dg_get_device_error(int* code);

/* Failure-detection self-test: launches one CTA that waits on an mbarrier
 * nothing ever completes.  The kernels' bounded wait gives up after about one
 * second, sets DG_DEVERR_TIMEOUT in the device error word and returns, so the
 * context stays usable.  Enqueued on `stream`; read the outcome with
 * dg_get_device_error().  Diagnostic only (no counterpart on the pages). */
DG_API dg_status dg_selftest_bounded_wait(void* stream);

/* Static text for a status code. */
DG_API const char* dg_status_string(dg_status s);
/* Text describing the last failing call on this host thread ("" if none). */
DG_API const char* dg_last_error_message(void);

/*
 * Launch plan (host only, no GPU needed; no counterpart on the pages): what a
 * call with these sizes would launch.  mode: 0 dense, 1 contiguous, 2
 * masked.  rows = M (dense), M_total (contiguous) or M_max (masked).
 * Returns DG_ERR_INVALID_ARG for bad sizes.
 */
typedef struct dg_plan {
    int block_m;      /* output rows per tile                                    */
    int block_n;      /* output columns per tile                                 */
    int stages;       /* depth of the shared-memory operand ring                 */
    int m_blocks;     /* tiles along M (masked: worst case, G*ceil(M_max/block_m)) */
    int n_blocks;     /* tiles along N                                           */
    int tiles;        /* m_blocks * n_blocks                                     */
    int grid;         /* CTAs launched                                           */
    int smem_bytes;   /* dynamic shared memory per CTA                           */
    int swap_ab;      /* 1: few-row kernel (weights on the MMA's 128-row side)   */
    int split_k;      /* CTAs (one thread-block cluster) sharing each tile's K   */
    int tail_split;   /* >1: the tiles of the last partial wave are split into   */
                      /* this many K slices (dense calls only; 1 = off)          */
} dg_plan;

DG_API dg_status dg_make_plan(int mode, int rows, int N, int K, int G, int num_sms, dg_plan* out);

/*
 * Launch plan (host only, no GPU needed; no counterpart on the pages) of the
 * block-scaled kernel that dg_fp8_gemm_nt_ue8m0 runs when it takes that
 * kernel (M > 256, or DG_FORCE_BLOCK_SCALED=1): 128 x 256 tiles, grid <=
 * num_sms, and tail_split > 1 when the tiles of the last partial wave (all
 * tiles, when there are fewer than num_sms; the grid is then tiles x
 * tail_split) are split along K.  swap_ab is 0 and split_k 1.  M == 0 gives
 * zero tiles.
 * Returns DG_ERR_INVALID_ARG / DG_ERR_UNSUPPORTED for the sizes
 * dg_fp8_gemm_nt_ue8m0 rejects, or for num_sms <= 0 or a null `out`.
 */
DG_API dg_status dg_make_plan_ue8m0(int M, int N, int K, int num_sms, dg_plan* out);

#ifdef __cplusplus
}
#endif

#endif /* DG_H_ */

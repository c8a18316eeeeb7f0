// dg_api.cu -- host side of the C ABI declared in include/dg.h: argument
// validation, the launch plan (tile shape, ring depth, grid), TMA tensor-map
// encoding and kernel dispatch.  Nothing here reads device memory or
// synchronises, except dg_get_device_error(); the only device allocation is
// the per-(device, stream) K-split workspace, made on first need (at most four
// streams per device keep one).
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdarg>
#include <cstdlib>
#include <cmath>
#include <map>
#include <utility>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "dg.h"
#include "dg_kernel.cuh"
#include "dg_kernel_small.cuh"
#include "dg_cast.cuh"
#include "dg_kernel_ue8m0.cuh"

namespace dg {
// One CTA waits (bounded) on a barrier that no one arrives at.
__global__ void bounded_wait_selftest_kernel() {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag);
}
}  // namespace dg

namespace {

thread_local char g_msg[512] = "";
std::atomic<int> g_num_sms_cap{0};

dg_status fail(dg_status s, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
    va_end(ap);
    return s;
}

dg_status ok() {
    g_msg[0] = '\0';
    return DG_OK;
}

int cdiv(int a, int b) { return (a + b - 1) / b; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ------------------------------------------------------------- devices ----

constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];

int device_sm_count(int* dev_out = nullptr) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    if (dev_out) *dev_out = dev;
    if (dev < 0 || dev >= kMaxDevices) return 0;
    int n = g_sm_count[dev].load();
    if (n == 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            cudaGetLastError();
            return 0;
        }
        g_sm_count[dev].store(n);
    }
    return n;
}

// ------------------------------------------------------ tensor maps ----

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        else
            cudaGetLastError();
    });
    return fn;
}

// K-major e4m3 operand: dims (K, rows[, groups]), box (128, box_rows[, 1]),
// 128-byte swizzle, zero fill outside the tensor.
dg_status make_operand_map(CUtensorMap* tm, const void* base, int K, int rows, int groups, int box_rows,
                           bool three_d) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(DG_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows),
                          static_cast<cuuint64_t>(groups)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(K) * rows};
    cuuint32_t box[3] = {static_cast<cuuint32_t>(dg::kBK), static_cast<cuuint32_t>(box_rows), 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, three_d ? 3 : 2, const_cast<void*>(base), dims, strides, box,
                    estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(DG_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", static_cast<int>(r));
    return DG_OK;
}

// MN-major operand stored [K][MN] (MN contiguous, MN % 16 == 0): dims (MN, K),
// box 128 (MN) x 128 (K) with 128-byte swizzle -- the canonical MN-major tile.
dg_status make_mn_operand_map(CUtensorMap* tm, const void* base, int MN, int K) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(DG_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(MN), static_cast<cuuint64_t>(K)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(MN)};
    cuuint32_t box[2] = {128, static_cast<cuuint32_t>(dg::kBK)};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(DG_ERR_CUDA, "cuTensorMapEncodeTiled (MN-major) failed (CUresult %d)", static_cast<int>(r));
    return DG_OK;
}

// bf16 output: dims (N, rows[, groups]), box (32, 32[, 1]) -- one promotion
// warp's 32 rows x 32 columns -- with 64-byte swizzle; the store clips
// everything outside the tensor.
dg_status make_output_map(CUtensorMap* tm, void* base, int N, int rows, int groups, bool three_d) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(DG_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(groups)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(N) * 2, static_cast<cuuint64_t>(N) * 2 * rows};
    cuuint32_t box[3] = {32, 32, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, three_d ? 3 : 2, base, dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(DG_ERR_CUDA, "cuTensorMapEncodeTiled (output) failed (CUresult %d)", static_cast<int>(r));
    return DG_OK;
}

// ------------------------------------------------------------ planning ----

struct Choice {
    int bn;
    int stages;
};

// Ring depth: as many stages as fit in 227 KiB of shared memory, at most 8.
template <int BN>
constexpr int max_stages() {
    int s = 8;
    while (s > 2 && dg::smem_bytes<BN, 8>() - (8 - s) * (dg::kTileABytes + BN * dg::kBK) > 227 * 1024) --s;
    return s;
}

int waves_cost(int tiles, int sms) { return cdiv(tiles, sms); }

template <int BN>
constexpr int smem_for() {
    return dg::smem_bytes<BN, max_stages<BN>()>();
}

// Tile width.  Each 128-wide K block costs a tile max(MMA time, operand
// streaming time): the tensor core's time grows with BN, while the bytes
// moved into shared memory are 16 KiB of A plus BN*128 B of B.  Relative
// units: MMA = BN, streaming = 0.75*(128 + BN).  The problem takes
// ceil(tiles / SMs) such tile times.  Narrower tiles win when they put more
// SMs to work -- the point of the "non-aligned block size" optimisation on
// the DeepGEMM README page (section "非对齐的块大小"); here BN stays a
// multiple of 64 so that the two promotion warpgroups split it into 32-column
// TMEM loads.
Choice choose(int m_blocks, int N, int num_sms, bool mn_major = false) {
    // An MN-major B is loaded in 128-wide atoms: tiles of 128 or 256 only.
    const int cands[3] = {256, 128, 64};
    Choice best{128, max_stages<128>()};
    double best_cost = -1.0;
    for (int bn : cands) {
        if (mn_major && bn % 128 != 0) continue;
        const int tiles = m_blocks * cdiv(N, bn);
        const double t_kb = bn > 0.75 * (128 + bn) ? bn : 0.75 * (128 + bn);
        const double cost = static_cast<double>(waves_cost(tiles, num_sms)) * t_kb;
        if (best_cost < 0 || cost < best_cost - 1e-9) {
            best_cost = cost;
            best.bn = bn;
        }
    }
    best.stages = best.bn == 256 ? max_stages<256>() : best.bn == 128 ? max_stages<128>() : max_stages<64>();
    return best;
}

// Dense NT calls of 128 x 256 tiles with at most kShortKBlocks K blocks per
// tile stage each promotion warp's whole epilogue at once (a 3-stage ring
// leaves room): with few K blocks per tile the epilogue is a large share of
// its time.
constexpr int kShortKBlocks = 16;
constexpr int kShortKStages = 3;

int plan_smem(const Choice& c) {
    return c.bn == 256 ? smem_for<256>() : c.bn == 128 ? smem_for<128>() : smem_for<64>();
}

dg_status check_sizes(int mode, int rows, int N, int K, int G) {
    if (rows < 0 || N <= 0 || K <= 0 || G <= 0)
        return fail(DG_ERR_INVALID_ARG, "sizes must be positive (rows=%d N=%d K=%d G=%d)", rows, N, K, G);
    if (K % 128 != 0) return fail(DG_ERR_UNSUPPORTED, "K=%d is not a multiple of 128", K);
    if (N % 8 != 0) return fail(DG_ERR_UNSUPPORTED, "N=%d is not a multiple of 8", N);
    if (mode == 1 && rows % dg::kBM != 0)
        return fail(DG_ERR_INVALID_ARG, "contiguous layout: M_total=%d is not a multiple of %d", rows, dg::kBM);
    if (mode == 2 && G > dg::kMaxMaskedGroups)
        return fail(DG_ERR_UNSUPPORTED, "masked layout supports at most %d groups (G=%d)", dg::kMaxMaskedGroups, G);
    const long long a_elems = static_cast<long long>(rows) * K * (mode == 2 ? G : 1);
    const long long b_elems = static_cast<long long>(mode == 3 ? 1 : G) * N * K;
    if (a_elems >= (1ll << 40) || b_elems >= (1ll << 40) || static_cast<long long>(rows) * G >= (1ll << 31))
        return fail(DG_ERR_UNSUPPORTED, "problem too large");
    return DG_OK;
}

// Few-row problems (dense M <= 128, masked M_max <= 256) go to the swap-AB
// kernel: 128 weight rows per tile, TN activation rows, one CTA per SM.
// Tiles are spread over clusters of S CTAs that split K; without a split the
// clusters are single CTAs that walk several tiles each.  small_choice picks
// TN and S.
bool use_small(int mode, int rows) { return (mode == 0 && rows <= 128) || (mode == 2 && rows <= 256); }

int small_tn(int mode, int rows) {
    const int t = rows < 128 ? rows : 128;
    return t <= 32 ? 32 : t <= 64 ? 64 : 128;
}

int small_max_split(int tn) {
    return tn == 32 ? dg::SmallCfg<32>::kMaxSplit : tn == 64 ? dg::SmallCfg<64>::kMaxSplit : dg::SmallCfg<128>::kMaxSplit;
}

// CTAs of clusters of `s` one-CTA-per-SM blocks that can be resident at once
// on `num_sms` SMs.  Clusters are placed inside GPCs, so large clusters leave
// SMs unused; measured on a 148-SM B200 with cudaOccupancyMaxActiveClusters
// (227 KiB of shared memory per CTA), scaled down for a smaller SM budget.
int small_cluster_capacity(int s, int num_sms) {
    static const int kB200[9] = {0, 148, 148, 135, 132, 130, 132, 105, 120};
    if (s < 1 || s > 8) return 0;
    const int cap = static_cast<int>(static_cast<long long>(kB200[s]) * num_sms / 148);
    return cap - cap % s;
}

// Estimated time (us) of a few-row launch with TN activation rows per tile
// and K split into `split` slices.  Fitted to CUDA-graph timings of the 12
// dense decode shapes of the sweep under 41 (TN, split) choices on a 148-SM
// B200 (rms error about 1 us); it picks the fastest measured choice, or one
// within 4 %, on every shape.  Terms: a fixed cost (launch, set-up, first
// loads); the longest CTA's K loop -- bound by its per-K-block pipeline cost,
// by its own operand stream (about 80 GB/s per CTA), or by the whole weight
// stream at HBM speed; the split reduction; an epilogue per tile.
double small_cost(long tiles, int nkb, int tn, int split, int num_sms, double weight_bytes) {
    constexpr double kFixedUs = 3.9, kReduceUs = 2.3, kTileUs = 0.58, kCtaGBs = 81.5, kHbmGBs = 6500.0;
    const double per_kb = tn == 32 ? 0.218 : tn == 64 ? 0.257 : 0.47;
    long kb_per_cta, tiles_per_cta;
    if (split > 1) {
        kb_per_cta = (nkb + split - 1) / split;
        tiles_per_cta = 1;
    } else {
        tiles_per_cta = (tiles + num_sms - 1) / num_sms;
        kb_per_cta = static_cast<long>(nkb) * tiles_per_cta;
    }
    const double loop = static_cast<double>(kb_per_cta) * per_kb;
    const double stream = static_cast<double>(kb_per_cta) * (128.0 + tn) * dg::kBK / (kCtaGBs * 1e3);
    const double hbm = weight_bytes / (kHbmGBs * 1e3);
    double t = loop > stream ? loop : stream;
    t = t > hbm ? t : hbm;
    return kFixedUs + t + (split > 1 ? kReduceUs : 0.0) + kTileUs * static_cast<double>(tiles_per_cta);
}

struct SmallChoice {
    int tn;
    int split;
};

// Tile height and K split of a few-row launch: the (TN, split) of least
// small_cost among TN in {32, 64, 128} no taller than the rows need (a
// shorter TN reads each weight tile once per TN-row block, from L2 after the
// first) and splits that keep at least kSmallMinSliceKb K blocks per slice,
// whose clusters all fit on the GPU at once, used only while the tiles alone
// leave SMs idle.  `rows` is the row count that decides the TN-row blocks
// (masked: the expected rows per group); `all_rows` the most a group can
// have, which the launch must cover.
SmallChoice small_choice(int rows, int all_rows, int G, int N, int K, int num_sms) {
    constexpr int kSmallMinSliceKb = 4;
    const int nkb = K / dg::kBK;
    const int n_blocks = cdiv(N, 128);
    const double weight_bytes = static_cast<double>(G) * N * K;
    const int tn_max = small_tn(0, all_rows);
    SmallChoice best{tn_max, 1};
    double best_t = -1.0;
    for (int tn = tn_max; tn >= 32; tn /= 2) {
        const long tiles = static_cast<long>(G) * cdiv(rows, tn) * n_blocks;
        const long all_tiles = static_cast<long>(G) * cdiv(all_rows, tn) * n_blocks;
        for (int split = 1; split <= small_max_split(tn); ++split) {
            if (split > 1 && (all_tiles >= num_sms || nkb / split < kSmallMinSliceKb ||
                              all_tiles * split > small_cluster_capacity(split, num_sms)))
                continue;
            const double t = small_cost(tiles, nkb, tn, split, num_sms, weight_bytes);
            if (best_t < 0 || t < best_t - 1e-9) {
                best_t = t;
                best = {tn, split};
            }
        }
    }
    return best;
}

int small_smem(int tn) {
    return tn == 32 ? dg::small_smem_bytes<32>() : tn == 64 ? dg::small_smem_bytes<64>() : dg::small_smem_bytes<128>();
}

int small_stages(int tn) {
    return tn == 32 ? dg::SmallCfg<32>::kStages : tn == 64 ? dg::SmallCfg<64>::kStages : dg::SmallCfg<128>::kStages;
}

dg_status plan(int mode, int rows, int N, int K, int G, int num_sms, dg_plan* out, int expected_m = 0,
               int layout = 0) {
    dg_status s = check_sizes(mode, rows, N, K, G);
    if (s != DG_OK) return s;
    if (num_sms <= 0) return fail(DG_ERR_INVALID_ARG, "num_sms must be positive");
    *out = dg_plan{};
    if (layout == 0 && use_small(mode, rows)) {
        // Masked: tiles past masked_m are skipped on the device; with a hint,
        // count only the tiles expected to hold rows.
        const int expect = (mode == 2 && expected_m > 0 && expected_m < rows) ? expected_m : rows;
        const SmallChoice ch = small_choice(expect, rows, mode == 2 ? G : 1, N, K, num_sms);
        const int tn = ch.tn, split = ch.split;
        const int per_group = cdiv(rows, tn);
        const int m_blocks = mode == 2 ? G * per_group : per_group;
        const int n_blocks = cdiv(N, 128);
        out->block_m = tn;
        out->block_n = 128;
        out->stages = small_stages(tn);
        out->m_blocks = m_blocks;
        out->n_blocks = n_blocks;
        out->tiles = m_blocks * n_blocks;
        // Split: one cluster per tile (the host tile count is an upper bound
        // of the device's for masked calls).  Unsplit: persistent, at most
        // one CTA per SM.
        const long all = static_cast<long>(m_blocks) * n_blocks;
        out->grid = split > 1 ? static_cast<int>(all * split) : static_cast<int>(all < num_sms ? all : num_sms);
        out->smem_bytes = small_smem(tn);
        out->swap_ab = 1;
        out->split_k = split;
        out->tail_split = 1;  // the cluster split replaces the tail split
        return DG_OK;
    }
    const int m_blocks = (mode == 2) ? G * cdiv(rows, dg::kBM) : cdiv(rows, dg::kBM);
    const Choice c = choose(m_blocks, N, num_sms, layout != 0);
    out->block_m = dg::kBM;
    out->block_n = c.bn;
    out->stages = c.stages;
    out->m_blocks = m_blocks;
    out->n_blocks = cdiv(N, c.bn);
    out->tiles = m_blocks * out->n_blocks;
    out->grid = (mode == 2) ? num_sms : (out->tiles < num_sms ? out->tiles : num_sms);
    out->smem_bytes = plan_smem(c);
    if (mode == 0 && layout == 0 && c.bn == 256 && K / dg::kBK <= kShortKBlocks) {
        out->stages = kShortKStages;
        out->smem_bytes = dg::smem_bytes<256, kShortKStages, 4>();
    }
    out->swap_ab = 0;
    out->split_k = 1;
    out->tail_split = 1;
    // Dense: when the last wave is partial (R leftover tiles after W full
    // waves), split each leftover tile into S K slices run by the idle CTAs.
    // A slice takes ~nkb/S K blocks; slice 0 then reads S-1 partial tiles
    // (each costs about 1.5 K blocks' time), so S ~ sqrt(nkb / 1.5) balances
    // the two; also S*R <= grid, S <= 8 and at least 16 K blocks per slice.
    if (mode == 0) {
        const int waves = out->tiles / out->grid;
        const int rest = out->tiles - waves * out->grid;
        const int nkb = K / dg::kBK;
        if (waves >= 1 && rest > 0) {
            int split = static_cast<int>(std::sqrt(nkb / 1.5) + 0.5);
            if (split > out->grid / rest) split = out->grid / rest;
            if (split > 8) split = 8;
            // Slices shorter than 16 K blocks do not repay the partial
            // write, the flag hand-off and the reduction (measured).
            if (split > nkb / 16) split = nkb / 16;
            if (split >= 2) out->tail_split = split;
        }
    }
    return DG_OK;
}

// ------------------------------------------------------------ launch ----

// Every launch allows programmatic dependent launch unless DG_PDL=0 (or
// dg_set_pdl(0)): the kernel's set-up (barriers, TMEM, tensor-map prefetch)
// may overlap the end of the previous kernel in the stream; the kernels always
// wait (griddepcontrol.wait) before touching global data.  Measured in
// CUDA-graph replays of back-to-back GEMMs it saves about 1 us per decode-sized
// launch (e.g. 64x32768x512: 9.7 -> 8.2 us) and 1-2 % on the large shapes;
// every GEMM kernel takes one CTA per SM, so a dependent grid's CTAs start on
// SMs as the previous grid leaves them.
std::atomic<int> g_pdl{-1};  // -1: from DG_PDL, else 0 / 1 from dg_set_pdl

bool pdl_enabled() {
    const int set = g_pdl.load();
    if (set >= 0) return set != 0;
    const char* v = std::getenv("DG_PDL");
    return !(v && v[0] == '0');
}

void set_pdl(cudaLaunchAttribute& a) {
    a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    a.val.programmaticStreamSerializationAllowed = pdl_enabled() ? 1 : 0;
}

template <int BN, int STAGES, int MODE, int LAYOUT = 0, int SP = 1>
dg_status launch_one(const dg::Params& p, const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& td,
                     int grid, cudaStream_t stream) {
    constexpr int smem = dg::smem_bytes<BN, STAGES, SP>();
    static_assert(smem <= 227 * 1024, "shared memory budget exceeded");
    auto kern = dg::fp8_gemm_kernel<BN, STAGES, MODE, LAYOUT, SP>;
    static std::atomic<int> attr_set[kMaxDevices];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < kMaxDevices && !attr_set[dev].load()) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
            return fail(DG_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(cudaGetLastError()));
        using C = dg::Cfg<BN>;
        if (C::kSplitRegs) {
            // The setmaxnreg split draws on the registers the CTA is launched
            // with (its threads x the compiled register count); a build whose
            // count cannot cover it would wait forever in setmaxnreg, so it is
            // refused here, before any launch.
            constexpr int need = 128 * C::kRegsLow + 128 * C::kEpiWGs * C::kRegsHigh;
            cudaFuncAttributes fa{};
            if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess)
                return fail(DG_ERR_CUDA, "cudaFuncGetAttributes: %s", cudaGetErrorString(cudaGetLastError()));
            if (fa.numRegs * C::kThreadsC < need)
                return fail(DG_ERR_UNSUPPORTED, "GEMM kernel (BN=%d) compiled with %d registers per thread x %d "
                            "threads, its register split needs %d", BN, fa.numRegs, C::kThreadsC, need);
        }
        attr_set[dev].store(1);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
    cfg.blockDim = dim3(dg::Cfg<BN>::kThreadsC, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    set_pdl(attr[0]);
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, p, ta, tb, td);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return fail(DG_ERR_CUDA, "kernel launch failed: %s", cudaGetErrorString(e));
    return ok();
}

template <int TN, int MODE>
dg_status launch_small(const dg::Params& p, const CUtensorMap& ta, const CUtensorMap& tb, const dg_plan& pl,
                       cudaStream_t stream) {
    constexpr int smem = dg::small_smem_bytes<TN>();
    auto kern = dg::fp8_gemm_swapab_kernel<TN, MODE>;
    static std::atomic<int> attr_set[kMaxDevices];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < kMaxDevices && !attr_set[dev].load()) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
            return fail(DG_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(cudaGetLastError()));
        attr_set[dev].store(1);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(pl.grid), 1, 1);
    cfg.blockDim = dim3(dg::kSmallThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(pl.split_k);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    set_pdl(attr[1]);
    cfg.numAttrs = 2;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, p, ta, tb);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return fail(DG_ERR_CUDA, "kernel launch failed: %s", cudaGetErrorString(e));
    return ok();
}

template <int MODE>
dg_status dispatch_small(const dg_plan& pl, const dg::Params& p, const CUtensorMap& ta, const CUtensorMap& tb,
                         cudaStream_t stream) {
    switch (pl.block_m) {
        case 32: return launch_small<32, MODE>(p, ta, tb, pl, stream);
        case 64: return launch_small<64, MODE>(p, ta, tb, pl, stream);
        case 128: return launch_small<128, MODE>(p, ta, tb, pl, stream);
        default: return fail(DG_ERR_UNSUPPORTED, "no few-row kernel for block_m=%d", pl.block_m);
    }
}

template <int MODE>
dg_status dispatch(const dg_plan& pl, const dg::Params& p, const CUtensorMap& ta, const CUtensorMap& tb,
                   const CUtensorMap& td, cudaStream_t stream) {
    switch (pl.block_n) {
        case 256:
            if (MODE == dg::kDense && pl.stages == kShortKStages)
                return launch_one<256, kShortKStages, MODE, 0, 4>(p, ta, tb, td, pl.grid, stream);
            return launch_one<256, max_stages<256>(), MODE>(p, ta, tb, td, pl.grid, stream);
        case 128: return launch_one<128, max_stages<128>(), MODE>(p, ta, tb, td, pl.grid, stream);
        case 64: return launch_one<64, max_stages<64>(), MODE>(p, ta, tb, td, pl.grid, stream);
        default: return fail(DG_ERR_UNSUPPORTED, "no kernel for block_n=%d", pl.block_n);
    }
}

template <int LAYOUT>
dg_status dispatch_layout(const dg_plan& pl, const dg::Params& p, const CUtensorMap& ta, const CUtensorMap& tb,
                          const CUtensorMap& td, cudaStream_t stream) {
    switch (pl.block_n) {
        case 256: return launch_one<256, max_stages<256>(), dg::kDense, LAYOUT>(p, ta, tb, td, pl.grid, stream);
        case 128: return launch_one<128, max_stages<128>(), dg::kDense, LAYOUT>(p, ta, tb, td, pl.grid, stream);
        default: return fail(DG_ERR_UNSUPPORTED, "no MN-major kernel for block_n=%d", pl.block_n);
    }
}

int effective_sms() {
    const int dev_sms = device_sm_count();
    const int cap = g_num_sms_cap.load();
    if (cap > 0 && (dev_sms == 0 || cap < dev_sms)) return cap;
    return dev_sms;
}

dg_status common_checks(const void* D, const void* A, const float* sa, int sa_stride, const void* B, const float* sb,
                        int rows) {
    if (!D || !A || !sa || !B || !sb) return fail(DG_ERR_INVALID_ARG, "null tensor pointer");
    if (!aligned16(D) || !aligned16(A) || !aligned16(sa) || !aligned16(B) || !aligned16(sb))
        return fail(DG_ERR_MISALIGNED, "tensor pointers must be 16-byte aligned");
    if (sa_stride < rows || sa_stride % 4 != 0)
        return fail(DG_ERR_INVALID_ARG, "sa_stride=%d must be >= %d and a multiple of 4", sa_stride, rows);
    return DG_OK;
}

// Raster group (m-blocks whose tiles run together, m fastest): B is streamed
// from HBM once per group, so the group should be as tall as possible while
// the group's A rows plus the weight tiles in flight across the grid
// (grid / group of them) still fit in L2 (budget 96 MiB of the 126 MB).
int choose_raster(int m_blocks, int n_blocks, int block_m, int block_n, int K, int grid) {
    const double budget = 96.0 * 1024 * 1024;
    int best = 1;
    for (int gm = 1; gm <= m_blocks; gm *= 2) {
        const double a_bytes = static_cast<double>(gm) * block_m * K;
        const int active_n = n_blocks < cdiv(grid, gm) ? n_blocks : cdiv(grid, gm);
        const double b_bytes = static_cast<double>(active_n) * block_n * K;
        if (a_bytes + b_bytes <= budget) best = gm;
    }
    return best;
}

// Workspace for the K-split tail: per (device, stream), allocated on first
// need, never during stream capture.  Holds one 128 x 256 FP32 partial per SM
// (the split keeps fewer than grid <= SMs partials) and their flags.  At most
// kMaxTailWorkspaces streams per device keep one: the first call on a further
// stream frees the least recently used (cudaFree waits for the whole device,
// so no launch still uses it).  Allocation and freeing run in relaxed capture
// mode, so that another thread's CUDA-graph capture is not invalidated; if
// either fails the call runs without the split (same result up to FP32
// summation order).
constexpr int kMaxTailWorkspaces = 4;

struct TailWorkspace {
    float* partials = nullptr;
    unsigned int* flags = nullptr;
    size_t flag_bytes = 0;
    uint64_t last_use = 0;
};

std::mutex g_ws_mu;
std::map<std::pair<int, cudaStream_t>, TailWorkspace> g_ws;
uint64_t g_ws_clock = 0;

// Allocation / free helpers for the workspace: relaxed capture mode for the
// calling thread, restored afterwards.
struct RelaxedCapture {
    cudaStreamCaptureMode prev = cudaStreamCaptureModeRelaxed;
    RelaxedCapture() { cudaThreadExchangeStreamCaptureMode(&prev); }
    ~RelaxedCapture() { cudaThreadExchangeStreamCaptureMode(&prev); }
};

bool tail_workspace(cudaStream_t stream, TailWorkspace* out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    std::lock_guard<std::mutex> lock(g_ws_mu);
    auto key = std::make_pair(dev, stream);
    auto it = g_ws.find(key);
    if (it != g_ws.end()) {
        it->second.last_use = ++g_ws_clock;
        *out = it->second;
        return true;
    }
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    if (cs != cudaStreamCaptureStatusNone) return false;
    const int sms = device_sm_count();
    if (sms <= 0) return false;
    RelaxedCapture relaxed;
    int on_dev = 0;
    auto lru = g_ws.end();
    for (auto j = g_ws.begin(); j != g_ws.end(); ++j) {
        if (j->first.first != dev) continue;
        ++on_dev;
        if (lru == g_ws.end() || j->second.last_use < lru->second.last_use) lru = j;
    }
    if (on_dev >= kMaxTailWorkspaces) {
        if (cudaFree(lru->second.partials) != cudaSuccess || cudaFree(lru->second.flags) != cudaSuccess) {
            cudaGetLastError();
            return false;
        }
        g_ws.erase(lru);
    }
    TailWorkspace ws;
    const size_t part_bytes = static_cast<size_t>(sms) * dg::kBM * 256 * sizeof(float);
    ws.flag_bytes = static_cast<size_t>(sms) * sizeof(unsigned int);
    if (cudaMalloc(&ws.partials, part_bytes) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    if (cudaMalloc(&ws.flags, ws.flag_bytes) != cudaSuccess || cudaMemset(ws.flags, 0, ws.flag_bytes) != cudaSuccess) {
        cudaGetLastError();
        cudaFree(ws.partials);
        return false;
    }
    ws.last_use = ++g_ws_clock;
    g_ws[key] = ws;
    *out = ws;
    return true;
}

// After a bounded wait ran out, a late slice may have raised a ready flag
// that no launch consumes; clear every workspace flag on the current device
// (the caller has synchronised it).
void clear_workspace_flags() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return;
    }
    std::lock_guard<std::mutex> lock(g_ws_mu);
    for (auto& kv : g_ws)
        if (kv.first.first == dev && cudaMemset(kv.second.flags, 0, kv.second.flag_bytes) != cudaSuccess)
            cudaGetLastError();
}

int tail_workspace_count() {
    std::lock_guard<std::mutex> lock(g_ws_mu);
    return static_cast<int>(g_ws.size());
}

dg::Params make_params(uint16_t* D, const float* sa, int sa_stride, const float* sb, int rows, int N, int K, int G,
                       const dg_plan& pl) {
    dg::Params p{};
    p.D = D;
    p.sa = sa;
    p.sb = sb;
    p.sa_stride = sa_stride;
    p.M = rows;
    p.N = N;
    p.K = K;
    p.G = G;
    p.nkb = K / dg::kBK;
    p.nbn = cdiv(N, 128);
    p.n_blocks = pl.n_blocks;
    p.m_blocks = pl.m_blocks;
    p.raster = pl.swap_ab ? 1
                          : choose_raster(pl.m_blocks, pl.n_blocks, pl.block_m, pl.block_n, K,
                                          pl.grid);
    p.b_stream = 0;
    p.tail_split = 1;
    p.full_tiles = pl.tiles;
    return p;
}

// Dense GEMM with the operands in any of the four storage orders (bit 0 of
// `layout`: A stored [K][M]; bit 1: B stored [K][N]).
dg_status gemm_layout(int layout, uint16_t* D, const uint8_t* A, const float* sa, int sa_stride, const uint8_t* B,
                      const float* sb, int M, int N, int K, void* stream) {
    dg_status s = check_sizes(0, M, N, K, 1);
    if (s != DG_OK) return s;
    if ((s = common_checks(D, A, sa, sa_stride, B, sb, M)) != DG_OK) return s;
    if ((layout & 1) && M % 16 != 0) return fail(DG_ERR_UNSUPPORTED, "A stored [K][M] needs M %% 16 == 0 (M=%d)", M);
    if ((layout & 2) && N % 16 != 0) return fail(DG_ERR_UNSUPPORTED, "B stored [K][N] needs N %% 16 == 0 (N=%d)", N);
    if (M == 0) return ok();
    const int sms = effective_sms();
    if (sms <= 0) return fail(DG_ERR_CUDA, "no CUDA device");
    dg_plan pl;
    if ((s = plan(0, M, N, K, 1, sms, &pl, 0, layout)) != DG_OK) return s;
    CUtensorMap ta, tb, td;
    if ((s = (layout & 1) ? make_mn_operand_map(&ta, A, M, K) : make_operand_map(&ta, A, K, M, 1, dg::kBM, false)) !=
        DG_OK)
        return s;
    if ((s = (layout & 2) ? make_mn_operand_map(&tb, B, N, K) : make_operand_map(&tb, B, K, N, 1, pl.block_n, true)) !=
        DG_OK)
        return s;
    if ((s = make_output_map(&td, D, N, M, 1, false)) != DG_OK) return s;
    dg::Params p = make_params(D, sa, sa_stride, sb, M, N, K, 1, pl);
    p.b_stream = pl.m_blocks == 1;
    TailWorkspace ws;
    if (pl.tail_split > 1 && tail_workspace(static_cast<cudaStream_t>(stream), &ws)) {
        p.tail_split = pl.tail_split;
        p.full_tiles = (pl.tiles / pl.grid) * pl.grid;
        p.ws = ws.partials;
        p.ws_flags = ws.flags;
    }
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    switch (layout) {
        case 1: return dispatch_layout<1>(pl, p, ta, tb, td, st);
        case 2: return dispatch_layout<2>(pl, p, ta, tb, td, st);
        case 3: return dispatch_layout<3>(pl, p, ta, tb, td, st);
        default: return fail(DG_ERR_INVALID_ARG, "bad layout %d", layout);
    }
}

// K-grouped GEMM (A stored [K][M], B stored [K][N], group g owning K rows
// [k_offsets[g], k_offsets[g+1]), output D [G][M][N]).
dg_status k_grouped(uint16_t* D, const uint8_t* A, const float* sa, int sa_stride, const uint8_t* B,
                    const float* sb, const int32_t* k_offsets, int G, int M, int N, int K, void* stream) {
    if (G <= 0 || M < 0 || N <= 0 || K <= 0)
        return fail(DG_ERR_INVALID_ARG, "sizes must be positive (G=%d M=%d N=%d K=%d)", G, M, N, K);
    dg_status s = check_sizes(3, M, N, K, G);
    if (s != DG_OK) return s;
    if ((s = common_checks(D, A, sa, sa_stride, B, sb, M)) != DG_OK) return s;
    if (!k_offsets) return fail(DG_ERR_INVALID_ARG, "null k_offsets");
    if (M % 16 != 0) return fail(DG_ERR_UNSUPPORTED, "A stored [K][M] needs M %% 16 == 0 (M=%d)", M);
    if (N % 16 != 0) return fail(DG_ERR_UNSUPPORTED, "B stored [K][N] needs N %% 16 == 0 (N=%d)", N);
    if (static_cast<long long>(G) * M >= (1ll << 31)) return fail(DG_ERR_UNSUPPORTED, "problem too large");
    if (M == 0) return ok();
    const int sms = effective_sms();
    if (sms <= 0) return fail(DG_ERR_CUDA, "no CUDA device");
    const int m_blocks = cdiv(M, dg::kBM);
    const Choice c = choose(G * m_blocks, N, sms, true);
    dg_plan pl{};
    pl.block_m = dg::kBM;
    pl.block_n = c.bn;
    pl.stages = c.stages;
    pl.m_blocks = m_blocks;
    pl.n_blocks = cdiv(N, c.bn);
    pl.tiles = G * m_blocks * pl.n_blocks;
    pl.grid = pl.tiles < sms ? pl.tiles : sms;
    pl.smem_bytes = plan_smem(c);
    pl.split_k = 1;
    pl.tail_split = 1;
    CUtensorMap ta, tb, td;
    if ((s = make_mn_operand_map(&ta, A, M, K)) != DG_OK) return s;
    if ((s = make_mn_operand_map(&tb, B, N, K)) != DG_OK) return s;
    if ((s = make_output_map(&td, D, N, M, G, true)) != DG_OK) return s;
    dg::Params p = make_params(D, sa, sa_stride, sb, M, N, K, G, pl);
    p.k_offsets = k_offsets;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    switch (pl.block_n) {
        case 256: return launch_one<256, max_stages<256>(), dg::kKGrouped, 3>(p, ta, tb, td, pl.grid, st);
        case 128: return launch_one<128, max_stages<128>(), dg::kKGrouped, 3>(p, ta, tb, td, pl.grid, st);
        default: return fail(DG_ERR_UNSUPPORTED, "no K-grouped kernel for block_n=%d", pl.block_n);
    }
}

}  // namespace

// ------------------------------------------------ allocation-free dense ----
// dg_fp8_gemm_nt_noalloc keeps the K-split tail's scratch in this fixed
// array instead of a workspace from cudaMalloc: FP32 partials in the first
// 16 MiB (128 tiles of 128 x 256), then 1024 ready flags.  The array is zero
// at module load and every GPU that loads the library holds it until the
// process exits.  All calls on a GPU share it.
constexpr size_t kNoAllocPartialBytes = size_t(16) << 20;
constexpr size_t kNoAllocFlags = 1024;
static __device__ __align__(256) unsigned char dg_noalloc_scratch[kNoAllocPartialBytes +
                                                                  kNoAllocFlags * sizeof(unsigned int)];

namespace {

// Device address of dg_noalloc_scratch on the current device.  On the host the
// symbol is only a handle, so the address is looked up once per device (with
// that device current) and cached.
dg_status noalloc_scratch(unsigned char** out) {
    static std::mutex mu;
    static std::map<int, unsigned char*> addrs;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(DG_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    }
    std::lock_guard<std::mutex> lock(mu);
    auto it = addrs.find(dev);
    if (it == addrs.end()) {
        unsigned char* ptr = nullptr;
        e = cudaGetSymbolAddress((void**)&ptr, dg_noalloc_scratch);
        if (e != cudaSuccess || ptr == nullptr) {
            cudaGetLastError();
            return fail(DG_ERR_CUDA, "cudaGetSymbolAddress(dg_noalloc_scratch) on device %d: %s", dev,
                        cudaGetErrorString(e));
        }
        it = addrs.emplace(dev, ptr).first;
    }
    *out = it->second;
    return DG_OK;
}

}  // namespace

extern "C" {

dg_status dg_fp8_gemm_nt(uint16_t* D, const uint8_t* A, const float* sa, int sa_stride, const uint8_t* B,
                         const float* sb, int M, int N, int K, void* stream) {
    dg_status s = check_sizes(0, M, N, K, 1);
    if (s != DG_OK) return s;
    if ((s = common_checks(D, A, sa, sa_stride, B, sb, M)) != DG_OK) return s;
    if (M == 0) return ok();
    const int sms = effective_sms();
    if (sms <= 0) return fail(DG_ERR_CUDA, "no CUDA device");
    dg_plan pl;
    if ((s = plan(0, M, N, K, 1, sms, &pl)) != DG_OK) return s;
    CUtensorMap ta, tb;
    if (pl.swap_ab) {
        if ((s = make_operand_map(&ta, A, K, M, 1, pl.block_m, false)) != DG_OK) return s;
        if ((s = make_operand_map(&tb, B, K, N, 1, 128, true)) != DG_OK) return s;
        dg::Params p = make_params(D, sa, sa_stride, sb, M, N, K, 1, pl);
        p.b_stream = pl.m_blocks == 1;
        return dispatch_small<dg::kDense>(pl, p, ta, tb, static_cast<cudaStream_t>(stream));
    }
    if ((s = make_operand_map(&ta, A, K, M, 1, dg::kBM, false)) != DG_OK) return s;
    if ((s = make_operand_map(&tb, B, K, N, 1, pl.block_n, true)) != DG_OK) return s;
    CUtensorMap td;
    if ((s = make_output_map(&td, D, N, M, 1, false)) != DG_OK) return s;
    dg::Params p = make_params(D, sa, sa_stride, sb, M, N, K, 1, pl);
    p.b_stream = pl.m_blocks == 1;
    TailWorkspace ws;
    if (pl.tail_split > 1 && tail_workspace(static_cast<cudaStream_t>(stream), &ws)) {
        p.tail_split = pl.tail_split;
        p.full_tiles = (pl.tiles / pl.grid) * pl.grid;
        p.ws = ws.partials;
        p.ws_flags = ws.flags;
    }
    return dispatch<dg::kDense>(pl, p, ta, tb, td, static_cast<cudaStream_t>(stream));
}

dg_status dg_fp8_gemm_nt_noalloc(uint16_t* D, const uint8_t* A, const float* sa, int sa_stride, const uint8_t* B,
                                 const float* sb, int M, int N, int K, void* stream) {
    dg_status s = check_sizes(0, M, N, K, 1);
    if (s != DG_OK) return s;
    if ((s = common_checks(D, A, sa, sa_stride, B, sb, M)) != DG_OK) return s;
    if (M == 0) return ok();
    unsigned char* scratch = nullptr;
    if ((s = noalloc_scratch(&scratch)) != DG_OK) return s;
    const int sms = effective_sms();
    if (sms <= 0) return fail(DG_ERR_CUDA, "no CUDA device");
    dg_plan pl;
    if ((s = plan(0, M, N, K, 1, sms, &pl)) != DG_OK) return s;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    CUtensorMap ta, tb;
    if (pl.swap_ab) {
        if ((s = make_operand_map(&ta, A, K, M, 1, pl.block_m, false)) != DG_OK) return s;
        if ((s = make_operand_map(&tb, B, K, N, 1, 128, true)) != DG_OK) return s;
        dg::Params p = make_params(D, sa, sa_stride, sb, M, N, K, 1, pl);
        p.b_stream = pl.m_blocks == 1;
        return dispatch_small<dg::kDense>(pl, p, ta, tb, st);
    }
    if ((s = make_operand_map(&ta, A, K, M, 1, dg::kBM, false)) != DG_OK) return s;
    if ((s = make_operand_map(&tb, B, K, N, 1, pl.block_n, true)) != DG_OK) return s;
    CUtensorMap td;
    if ((s = make_output_map(&td, D, N, M, 1, false)) != DG_OK) return s;
    dg::Params p = make_params(D, sa, sa_stride, sb, M, N, K, 1, pl);
    p.b_stream = pl.m_blocks == 1;
    if (pl.tail_split > 1) {
        // One partial per (tail tile, slice >= 1) and one flag per partial.
        const int full = (pl.tiles / pl.grid) * pl.grid;
        const size_t slots = static_cast<size_t>(pl.tiles - full) * (pl.tail_split - 1);
        const size_t part_bytes = slots * dg::kBM * pl.block_n * sizeof(float);
        if (part_bytes > kNoAllocPartialBytes || slots > kNoAllocFlags)
            return fail(DG_ERR_UNSUPPORTED,
                        "dg_fp8_gemm_nt_noalloc: M=%d N=%d K=%d on %d SMs needs %zu bytes of K-split partials "
                        "and %zu flags; the static scratch holds %zu bytes and %zu flags",
                        M, N, K, pl.grid, part_bytes, slots, kNoAllocPartialBytes, kNoAllocFlags);
        unsigned int* flags = reinterpret_cast<unsigned int*>(scratch + kNoAllocPartialBytes);
        // The flags must start at zero; a previous call that gave up on a wait
        // may have left some set.  The partials are always written before read.
        const cudaError_t e = cudaMemsetAsync(flags, 0, slots * sizeof(unsigned int), st);
        if (e != cudaSuccess) {
            cudaGetLastError();
            return fail(DG_ERR_CUDA, "clearing the scratch flags: %s", cudaGetErrorString(e));
        }
        p.tail_split = pl.tail_split;
        p.full_tiles = full;
        p.ws = reinterpret_cast<float*>(scratch);
        p.ws_flags = flags;
    }
    return dispatch<dg::kDense>(pl, p, ta, tb, td, st);
}

// K-split of the block-scaled kernel: the R tiles left after the full waves
// (all tiles when there are fewer than SMs) are each split into S K slices
// run by otherwise idle CTAs.  The rule is the promotion kernel's tail split:
// S ~ sqrt(nkb / 1.5) balances a slice's K blocks against slice 0's
// reduction of S-1 partials; S*R <= SMs, S <= 8, and at least 16 K blocks
// per slice.  Returns 1 for no split.
static int ue8m0_split(int tiles, int nkb, int sms) {
    const int rest = tiles % sms;
    if (rest == 0) return 1;
    int split = static_cast<int>(std::sqrt(nkb / 1.5) + 0.5);
    if (split > sms / rest) split = sms / rest;
    if (split > 8) split = 8;
    if (split > nkb / 16) split = nkb / 16;
    return split >= 2 ? split : 1;
}

// Launch plan of the block-scaled kernel: 128 x kUeBN tiles, persistent on
// at most `sms` CTAs, plus the K-split above (with fewer tiles than SMs,
// every tile is split and the grid is tiles x split).
static void ue8m0_plan(int M, int N, int K, int sms, dg_plan* pl) {
    *pl = dg_plan{};
    pl->block_m = dg::kBM;
    pl->block_n = dg::kUeBN;
    pl->stages = dg::kUeStages;
    pl->m_blocks = cdiv(M, dg::kBM);
    pl->n_blocks = cdiv(N, dg::kUeBN);
    pl->tiles = pl->m_blocks * pl->n_blocks;
    pl->grid = pl->tiles < sms ? pl->tiles : sms;
    pl->smem_bytes = dg::ue8m0_smem_bytes();
    pl->split_k = 1;
    pl->tail_split = ue8m0_split(pl->tiles, K / dg::kBK, sms);
    if (pl->tail_split > 1 && pl->tiles < sms) pl->grid = pl->tiles * pl->tail_split;
}

dg_status dg_make_plan_ue8m0(int M, int N, int K, int num_sms, dg_plan* out) {
    if (!out) return fail(DG_ERR_INVALID_ARG, "null plan pointer");
    dg_status s = check_sizes(0, M, N, K, 1);
    if (s != DG_OK) return s;
    if (num_sms <= 0) return fail(DG_ERR_INVALID_ARG, "num_sms must be positive");
    ue8m0_plan(M, N, K, num_sms, out);
    return DG_OK;
}

dg_status dg_fp8_gemm_nt_ue8m0(uint16_t* D, const uint8_t* A, const float* sa, int sa_stride, const uint8_t* B,
                               const float* sb, int M, int N, int K, void* stream) {
    dg_status s = check_sizes(0, M, N, K, 1);
    if (s != DG_OK) return s;
    if ((s = common_checks(D, A, sa, sa_stride, B, sb, M)) != DG_OK) return s;
    if (M == 0) return ok();
    const int sms = effective_sms();
    if (sms <= 0) return fail(DG_ERR_CUDA, "no CUDA device");
    // Routing.  With the scale-factor conversion split over two warps and the
    // K-split of a partial last wave, the block-scaled kernel measured faster
    // than the promotion kernel on power-of-two scales (CUDA-graph replays on
    // B200) on every M = 4096 shape of the dense sweep, by 4 % (7168 x 16384)
    // to 25 % (32768 x 512), and 5 % slower at 256 x 7168 x 7168.  So M > 256
    // takes it; fewer rows go to the promotion path, whose few-row kernel
    // streams the weights with 32- or 64-row tiles.  DG_FORCE_BLOCK_SCALED=1
    // always takes the block-scaled kernel, =0 never.
    {
        const char* force = std::getenv("DG_FORCE_BLOCK_SCALED");
        bool block_scaled = M > 256;
        if (force && force[0] == '1') block_scaled = true;
        if (force && force[0] == '0') block_scaled = false;
        if (!block_scaled) return dg_fp8_gemm_nt(D, A, sa, sa_stride, B, sb, M, N, K, stream);
    }
    dg_plan pl;
    ue8m0_plan(M, N, K, sms, &pl);
    CUtensorMap ta, tb, td;
    if ((s = make_operand_map(&ta, A, K, M, 1, dg::kBM, false)) != DG_OK) return s;
    if ((s = make_operand_map(&tb, B, K, N, 1, dg::kUeBN, true)) != DG_OK) return s;
    if ((s = make_output_map(&td, D, N, M, 1, false)) != DG_OK) return s;
    dg::Params p = make_params(D, sa, sa_stride, sb, M, N, K, 1, pl);
    p.b_stream = pl.m_blocks == 1;
    TailWorkspace ws;
    if (pl.tail_split > 1 && tail_workspace(static_cast<cudaStream_t>(stream), &ws)) {
        p.tail_split = pl.tail_split;
        p.full_tiles = (pl.tiles / pl.grid) * pl.grid;
        p.ws = ws.partials;
        p.ws_flags = ws.flags;
    }
    constexpr int smem = dg::ue8m0_smem_bytes();
    static_assert(smem <= 227 * 1024, "shared memory budget exceeded");
    auto kern = dg::fp8_gemm_ue8m0_kernel;
    static std::atomic<int> attr_set[kMaxDevices];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < kMaxDevices && !attr_set[dev].load()) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
            return fail(DG_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(cudaGetLastError()));
        // The kernel's setmaxnreg split draws on the registers the CTA is
        // launched with (its threads x the compiled register count); a build
        // whose count cannot cover the split would wait forever in
        // setmaxnreg, so it is refused here, before any launch.
        cudaFuncAttributes fa{};
        if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess)
            return fail(DG_ERR_CUDA, "cudaFuncGetAttributes: %s", cudaGetErrorString(cudaGetLastError()));
        if (fa.numRegs < dg::kUeLaunchRegsNeeded)
            return fail(DG_ERR_UNSUPPORTED, "block-scaled kernel compiled with %d registers per thread, its register "
                        "split needs %d", fa.numRegs, dg::kUeLaunchRegsNeeded);
        attr_set[dev].store(1);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(pl.grid), 1, 1);
    cfg.blockDim = dim3(dg::kUeThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    set_pdl(attr[0]);
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, p, ta, tb, td);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return fail(DG_ERR_CUDA, "kernel launch failed: %s", cudaGetErrorString(e));
    return ok();
}

dg_status dg_fp8_gemm_nn(uint16_t* D, const uint8_t* A, const float* sa, int sa_stride, const uint8_t* B,
                         const float* sb, int M, int N, int K, void* stream) {
    return gemm_layout(2, D, A, sa, sa_stride, B, sb, M, N, K, stream);
}

dg_status dg_fp8_gemm_tn(uint16_t* D, const uint8_t* A, const float* sa, int sa_stride, const uint8_t* B,
                         const float* sb, int M, int N, int K, void* stream) {
    return gemm_layout(3, D, A, sa, sa_stride, B, sb, M, N, K, stream);
}

dg_status dg_fp8_gemm_tt(uint16_t* D, const uint8_t* A, const float* sa, int sa_stride, const uint8_t* B,
                         const float* sb, int M, int N, int K, void* stream) {
    return gemm_layout(1, D, A, sa, sa_stride, B, sb, M, N, K, stream);
}

dg_status dg_k_grouped_fp8_gemm_tn(uint16_t* D, const uint8_t* A, const float* sa, int sa_stride, const uint8_t* B,
                                   const float* sb, const int32_t* k_offsets, int G, int M, int N, int K,
                                   void* stream) {
    return k_grouped(D, A, sa, sa_stride, B, sb, k_offsets, G, M, N, K, stream);
}

dg_status dg_grouped_contiguous_nt(uint16_t* D, const uint8_t* A, const float* sa, int sa_stride, const uint8_t* B,
                                   const float* sb, const int32_t* m_indices, int M_total, int N, int K, int G,
                                   void* stream) {
    dg_status s = check_sizes(1, M_total, N, K, G);
    if (s != DG_OK) return s;
    if ((s = common_checks(D, A, sa, sa_stride, B, sb, M_total)) != DG_OK) return s;
    if (!m_indices) return fail(DG_ERR_INVALID_ARG, "null m_indices");
    if (M_total == 0) return ok();
    const int sms = effective_sms();
    if (sms <= 0) return fail(DG_ERR_CUDA, "no CUDA device");
    dg_plan pl;
    if ((s = plan(1, M_total, N, K, G, sms, &pl)) != DG_OK) return s;
    CUtensorMap ta, tb;
    if ((s = make_operand_map(&ta, A, K, M_total, 1, dg::kBM, false)) != DG_OK) return s;
    if ((s = make_operand_map(&tb, B, K, N, G, pl.block_n, true)) != DG_OK) return s;
    CUtensorMap td;
    if ((s = make_output_map(&td, D, N, M_total, 1, false)) != DG_OK) return s;
    dg::Params p = make_params(D, sa, sa_stride, sb, M_total, N, K, G, pl);
    p.m_indices = m_indices;
    return dispatch<dg::kContiguous>(pl, p, ta, tb, td, static_cast<cudaStream_t>(stream));
}

dg_status dg_grouped_masked_nt(uint16_t* D, const uint8_t* A, const float* sa, int sa_stride, const uint8_t* B,
                               const float* sb, const int32_t* masked_m, int G, int M_max, int N, int K,
                               int expected_m, void* stream) {
    dg_status s = check_sizes(2, M_max, N, K, G);
    if (s != DG_OK) return s;
    if ((s = common_checks(D, A, sa, sa_stride, B, sb, M_max)) != DG_OK) return s;
    if (!masked_m) return fail(DG_ERR_INVALID_ARG, "null masked_m");
    if (M_max == 0) return ok();
    const int sms = effective_sms();
    if (sms <= 0) return fail(DG_ERR_CUDA, "no CUDA device");
    dg_plan pl;
    if ((s = plan(2, M_max, N, K, G, sms, &pl, expected_m)) != DG_OK) return s;
    CUtensorMap ta, tb;
    if (pl.swap_ab) {
        if ((s = make_operand_map(&ta, A, K, M_max, G, pl.block_m, true)) != DG_OK) return s;
        if ((s = make_operand_map(&tb, B, K, N, G, 128, true)) != DG_OK) return s;
        dg::Params p = make_params(D, sa, sa_stride, sb, M_max, N, K, G, pl);
        p.masked_m = masked_m;
        p.m_blocks = pl.m_blocks / G;  // TN-row blocks per group
        p.b_stream = p.m_blocks == 1;
        return dispatch_small<dg::kMasked>(pl, p, ta, tb, static_cast<cudaStream_t>(stream));
    }
    if ((s = make_operand_map(&ta, A, K, M_max, G, dg::kBM, true)) != DG_OK) return s;
    if ((s = make_operand_map(&tb, B, K, N, G, pl.block_n, true)) != DG_OK) return s;
    CUtensorMap td;
    if ((s = make_output_map(&td, D, N, M_max, G, true)) != DG_OK) return s;
    dg::Params p = make_params(D, sa, sa_stride, sb, M_max, N, K, G, pl);
    p.masked_m = masked_m;
    p.b_stream = M_max <= dg::kBM;
    return dispatch<dg::kMasked>(pl, p, ta, tb, td, static_cast<cudaStream_t>(stream));
}

dg_status dg_to_fp8_1x128(uint8_t* Q, float* sa, int sa_stride, const uint16_t* X, int M, int K, void* stream) {
    if (M < 0 || K <= 0) return fail(DG_ERR_INVALID_ARG, "bad sizes M=%d K=%d", M, K);
    if (K % dg::kBK != 0) return fail(DG_ERR_UNSUPPORTED, "K=%d must be a multiple of 128", K);
    if (!Q || !sa || !X) return fail(DG_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(Q) || !aligned16(X) || (reinterpret_cast<uintptr_t>(sa) & 3u))
        return fail(DG_ERR_MISALIGNED, "X and Q must be 16-byte aligned, sa 4-byte aligned");
    if (sa_stride < M) return fail(DG_ERR_INVALID_ARG, "sa_stride=%d must be >= M=%d", sa_stride, M);
    if (M == 0) return ok();
    const int sms = effective_sms();
    if (sms <= 0) return fail(DG_ERR_CUDA, "no CUDA device");
    dg::CastParams p{Q, sa, X, M, K, K / dg::kBK, sa_stride};
    const int64_t items = static_cast<int64_t>(cdiv(M, dg::kCastRowsPerCta)) * cdiv(K / dg::kBK, dg::kCastBlocks);
    const int64_t cap = static_cast<int64_t>(sms) * 8;  // 8 CTAs of 256 threads per SM
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(items < cap ? items : cap), 1, 1);
    cfg.blockDim = dim3(dg::kCastThreads, 1, 1);
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    set_pdl(attr[0]);
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, dg::cast_1x128_kernel, p);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return fail(DG_ERR_CUDA, "kernel launch failed: %s", cudaGetErrorString(e));
    return ok();
}

dg_status dg_to_fp8_128x128(uint8_t* Q, float* sb, const uint16_t* W, int N, int K, void* stream) {
    if (N < 0 || K <= 0) return fail(DG_ERR_INVALID_ARG, "bad sizes N=%d K=%d", N, K);
    if (K % dg::kBK != 0) return fail(DG_ERR_UNSUPPORTED, "K=%d must be a multiple of 128", K);
    if (!Q || !sb || !W) return fail(DG_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(Q) || !aligned16(W) || (reinterpret_cast<uintptr_t>(sb) & 3u))
        return fail(DG_ERR_MISALIGNED, "W and Q must be 16-byte aligned, sb 4-byte aligned");
    if (N == 0) return ok();
    if (cdiv(N, 128) > 65535) return fail(DG_ERR_UNSUPPORTED, "N=%d too large", N);
    dg::CastParams p{Q, sb, W, N, K, K / dg::kBK, 0};
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(K / dg::kBK), static_cast<unsigned>(cdiv(N, 128)), 1);
    cfg.blockDim = dim3(dg::kCastThreads, 1, 1);
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    set_pdl(attr[0]);
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, dg::cast_128x128_kernel, p);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return fail(DG_ERR_CUDA, "kernel launch failed: %s", cudaGetErrorString(e));
    return ok();
}

void dg_set_pdl(int enable) { g_pdl.store(enable < 0 ? -1 : (enable ? 1 : 0)); }

int dg_get_pdl(void) { return pdl_enabled() ? 1 : 0; }

void dg_set_num_sms(int n) { g_num_sms_cap.store(n > 0 ? n : 0); }

int dg_get_num_sms(void) { return effective_sms(); }

int dg_get_m_alignment_for_contiguous_layout(void) { return dg::kBM; }

int dg_get_tma_aligned_size(int x, int elem_bytes) {
    if (x < 0 || elem_bytes <= 0 || 16 % elem_bytes != 0) return -1;
    const int per = 16 / elem_bytes;
    return cdiv(x, per) * per;
}

int dg_get_workspace_count(void) { return tail_workspace_count(); }

dg_status dg_get_device_error(int* code) {
    if (!code) return fail(DG_ERR_INVALID_ARG, "null code pointer");
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return fail(DG_ERR_CUDA, "cudaDeviceSynchronize: %s", cudaGetErrorString(e));
    unsigned int v = 0, zero = 0;
    e = cudaMemcpyFromSymbol(&v, dg::g_dg_error, sizeof(v));
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(dg::g_dg_error, &zero, sizeof(zero));
    if (e != cudaSuccess) return fail(DG_ERR_CUDA, "reading the device error word: %s", cudaGetErrorString(e));
    if (v & DG_DEVERR_TIMEOUT) clear_workspace_flags();
    *code = static_cast<int>(v);
    return ok();
}

dg_status dg_selftest_bounded_wait(void* stream) {
    dg::bounded_wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>();
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(DG_ERR_CUDA, "self-test launch failed: %s", cudaGetErrorString(e));
    return ok();
}

const char* dg_status_string(dg_status s) {
    switch (s) {
        case DG_OK: return "ok";
        case DG_ERR_INVALID_ARG: return "invalid argument";
        case DG_ERR_UNSUPPORTED: return "unsupported shape or layout";
        case DG_ERR_MISALIGNED: return "misaligned pointer";
        case DG_ERR_CUDA: return "CUDA error";
    }
    return "unknown status";
}

const char* dg_last_error_message(void) { return g_msg; }

dg_status dg_make_plan(int mode, int rows, int N, int K, int G, int num_sms, dg_plan* out) {
    if (!out) return fail(DG_ERR_INVALID_ARG, "null plan pointer");
    if (mode < 0 || mode > 2) return fail(DG_ERR_INVALID_ARG, "mode must be 0, 1 or 2");
    if (mode == 0 && G != 1) return fail(DG_ERR_INVALID_ARG, "dense mode needs G == 1");
    return plan(mode, rows, N, K, G, num_sms, out);
}

}  // extern "C"

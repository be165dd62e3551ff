// bqgemm.cu -- host side of libbqgemm: argument checks, the M-threshold
// dispatcher, TMA descriptor creation, kernel launches and the C ABI declared
// in include/bqgemm.h.  Built as one translation unit with the kernels.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <type_traits>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <vector>

#include "bqgemm.h"
#include "common.cuh"
#include "dequant.cuh"
#include "gemv.cuh"
#include "gemv_q8.cuh"
#include "gemv_affine.cuh"
#include "gemv_stream.cuh"
#include "tc_gemm.cuh"

namespace bq {
namespace {

constexpr int kMaxDevices = 64;
constexpr int kGemvMaxM = 32;

// ------------------------------------------------------------------ device info
struct DeviceInfo {
    bool ok = false;
    int num_sms = 0;
    int max_smem_optin = 0;
};

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];
bool g_dev_init[kMaxDevices] = {};

bq_status current_device(int* dev_out, DeviceInfo* info_out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return BQ_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_dev_init[dev]) {
        DeviceInfo di;
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&di.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&di.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
            return BQ_ERR_CUDA;
        di.ok = (major == 10 && minor == 0);
        g_dev[dev] = di;
        g_dev_init[dev] = true;
    }
    if (!g_dev[dev].ok) return BQ_ERR_DEVICE;
    *dev_out = dev;
    *info_out = g_dev[dev];
    return BQ_OK;
}

// ------------------------------------------------------------------ checks
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Q4_0, affine 4- and 8-bit (every path), affine 2-, 3- and 6-bit (dequantize,
// quantize, the decode GEMV up to kGaMaxM tokens and the unfused pair).
enum class WFmt { Q4_0, AFF4, AFF8, AFF2, AFF3, AFF6 };

bool has_fast_paths(WFmt f) { return f == WFmt::Q4_0 || f == WFmt::AFF4 || f == WFmt::AFF8; }

constexpr int64_t kGaMaxM = 8;   // tokens of one decode GEMV launch for 2-, 3- and 6-bit weights
constexpr int64_t kGaAutoMaxM = 8;     // ... that the dispatcher sends to it
constexpr int64_t kGaForcedMaxM = 32;  // ... that a forced BQ_PATH_GEMV takes (in passes of kGaMaxM)

// Format and shape checks shared by quant_matmul and its helpers (host only):
// the packed matrix has N rows of K codes, grouped along K.
bq_status check_format(const void* biases, int64_t N, int64_t K, int group_size, int bits, WFmt* fmt)
{
    if (N < 0 || K < 0) return BQ_ERR_SHAPE;
    if (biases == nullptr) {
        if (bits != 4 || group_size != 32) return BQ_ERR_UNSUPPORTED;
        if (K % 32 != 0) return BQ_ERR_SHAPE;
        *fmt = WFmt::Q4_0;
    } else {
        switch (bits) {
        case 2: *fmt = WFmt::AFF2; break;
        case 3: *fmt = WFmt::AFF3; break;
        case 4: *fmt = WFmt::AFF4; break;
        case 6: *fmt = WFmt::AFF6; break;
        case 8: *fmt = WFmt::AFF8; break;
        default: return BQ_ERR_UNSUPPORTED;
        }
        if (group_size != 32 && group_size != 64 && group_size != 128) return BQ_ERR_UNSUPPORTED;
        if (K % group_size != 0) return BQ_ERR_SHAPE;
    }
    return BQ_OK;
}

// check_format selects the format from the biases pointer; these stand in for
// it where only the format matters (no dereference).
const void* const kAffineTag = reinterpret_cast<const void*>(uintptr_t(16));

// Without a biases pointer the format is inferred: group_size 32 with 4 bits is
// Q4_0, anything else is affine.
const void* format_tag(int group_size, int bits)
{
    return (group_size == 32 && bits == 4) ? nullptr : kAffineTag;
}

bq_status launch_status()
{
    return cudaGetLastError() == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

int grid_for(int64_t items, int threads, const DeviceInfo& di)
{
    int64_t g = (items + threads - 1) / threads;
    g = std::min<int64_t>(g, (int64_t)di.num_sms * 16);
    return (int)std::max<int64_t>(g, 1);
}

// ------------------------------------------------------------------ env config
// Default fused/pair thresholds per format, from B200 sweeps of the 12288 x 4096
// projection at M = 256 .. 8192 (20 graph-captured calls per timing): the fused
// kernel leads up to 3072 tokens for Q4_0 and affine 4-bit (230 / 236 vs 243 us
// at 3072), ties or trails from 4096; for affine 8-bit it leads up to 1024 tokens
// and trails from 2048 (192 vs 182 us).
constexpr int64_t kDefaultPairMinM[3] = {4096, 4096, 2048};   // Q4_0, affine4, affine8
// Default GEMV/fused thresholds per format, from B200 sweeps of the same
// projection at M = 8 .. 32: the fused kernel stays near 21.1-21.8 us (Q4_0),
// 22.0-22.4 (affine 4-bit), 22.5-23.3 (affine 8-bit) while the GEMV grows with M;
// they meet at M = 20 for the 4-bit formats (21.8 / 21.7, 22.4 / 22.3 us) and
// between 12 and 16 for affine 8-bit (22.4-23.0 / 23.0 us at 16).
constexpr int kDefaultTcMinM[3] = {21, 21, 17};

struct DispatchCfg {
    int tc_min_m[3] = {kDefaultTcMinM[0], kDefaultTcMinM[1], kDefaultTcMinM[2]};
    int64_t pair_min_m[3] = {kDefaultPairMinM[0], kDefaultPairMinM[1], kDefaultPairMinM[2]};   // 0: never
};

const DispatchCfg& dispatch_cfg()
{
    static DispatchCfg cfg = [] {
        DispatchCfg c;
        if (const char* v = std::getenv("BQ_TC_MIN_M")) {
            long t = std::strtol(v, nullptr, 10);
            for (int f = 0; f < 3; ++f) c.tc_min_m[f] = (int)std::min<long>(std::max<long>(t, 1), kGemvMaxM + 1);
        }
        if (const char* v = std::getenv("BQ_PAIR_MIN_M")) {
            long long t = std::strtoll(v, nullptr, 10);
            for (int f = 0; f < 3; ++f) c.pair_min_m[f] = t > 0 ? t : 0;
        }
        return c;
    }();
    return cfg;
}

int select_path(int64_t M, int64_t K, WFmt fmt)
{
    if (!has_fast_paths(fmt)) return M <= kGaAutoMaxM ? BQ_PATH_GEMV : BQ_PATH_DEQUANT_GEMM;
    const DispatchCfg& c = dispatch_cfg();
    if (M < c.tc_min_m[(int)fmt]) return BQ_PATH_GEMV;
    if (M <= kGemvMaxM && K % 64 != 0) return BQ_PATH_GEMV;      // no fused tile: the GEMV, not the pair
    const int64_t pair_min = c.pair_min_m[(int)fmt];
    if (pair_min > 0 && M >= pair_min) return BQ_PATH_DEQUANT_GEMM;
    return (K % 64 == 0) ? BQ_PATH_TC_FUSED : BQ_PATH_DEQUANT_GEMM;
}

// ------------------------------------------------------------------ TMA descriptors
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            p = nullptr;
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

// Packed code rows [rows][row_bytes] seen as 3-D [row_bytes / 128][rows][128 bytes]
// (strides 128 and row_bytes bytes), box [chunks][16][128 bytes], 128-byte swizzle.
bool make_code_map_3d(CUtensorMap* m, const void* ptr, int64_t rows, int64_t row_bytes, int chunks)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t gdim[3] = {128, (cuuint64_t)rows, (cuuint64_t)(row_bytes / 128)};
    cuuint64_t gstride[2] = {(cuuint64_t)row_bytes, 128};
    cuuint32_t box[3] = {128, 16, (cuuint32_t)chunks};
    cuuint32_t estride[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), gdim, gstride, box, estride,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 16-bit scale rows [rows][groups] seen as 3-D [groups / 8][rows][8 values]
// (strides 16 and groups * 2 bytes), box [units][16][8 values], no swizzle: the
// rows of one 16-byte unit land 16 bytes apart.
bool make_scale_map_3d(CUtensorMap* m, const void* ptr, int64_t rows, int64_t groups, int units)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t gdim[3] = {8, (cuuint64_t)rows, (cuuint64_t)(groups / 8)};
    cuuint64_t gstride[2] = {(cuuint64_t)(groups * 2), 16};
    cuuint32_t box[3] = {8, 16, (cuuint32_t)units};
    cuuint32_t estride[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<void*>(ptr), gdim, gstride, box, estride,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Row-major 2-D [rows][cols] tensor, tile box [box_rows][box_cols].
bool make_map(CUtensorMap* m, CUtensorMapDataType dt, int elem_bytes, const void* ptr, int64_t rows, int64_t cols,
              int box_rows, int box_cols, CUtensorMapSwizzle sw)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t gstride[1] = {(cuuint64_t)(cols * elem_bytes)};
    cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
    cuuint32_t estride[2] = {1, 1};
    return fn(m, dt, 2, const_cast<void*>(ptr), gdim, gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ tensor-core GEMM
// Token tile bn (MMA N) for the persistent kernel: each CTA runs
// ceil(tiles / grid) tiles, each costing about bn + overhead (token units; the
// overhead stands for per-tile work independent of bn, e.g. dequantization).
int choose_bn(int64_t M, int64_t N, int num_sms, int max_bn, int overhead)
{
    const int64_t ntiles = (N + 127) / 128;
    int best_bn = 16;
    int64_t best_cost = INT64_MAX;
    for (int bn = 16; bn <= max_bn; bn += 16) {
        const int64_t tiles = ((M + bn - 1) / bn) * ntiles;
        const int64_t grid = std::min<int64_t>(tiles, num_sms);
        const int64_t rounds = (tiles + grid - 1) / grid;
        const int64_t cost = rounds * (bn + overhead);
        if (cost < best_cost || (cost == best_cost && bn > best_bn)) {
            best_cost = cost;
            best_bn = bn;
        }
        if (bn >= M) break;   // larger tiles only add padding
    }
    return best_bn;
}

// Launch plan of the tensor-core kernel for one problem on one device.
struct TcPlan {
    int bn = 0, num_acc = 2, acc_stride = 0, stages = 0, splits = 1;
    int64_t tiles = 0;
    int64_t dp_tiles = 0;     // tiles run whole; the rest are split `splits` ways
    size_t ws_bytes = 0;      // fp32 partials needed when splits > 1
};

// fp32 partial sums of the split tiles: one bn x 128 tile per split and tile
size_t splitk_ws_bytes(int splits, int64_t split_tiles, int bn)
{
    return splits > 1 ? (size_t)splits * (size_t)split_tiles * (size_t)bn * 128u * 4u : 0u;
}

template <int MODE>
bool plan_tc(int64_t M, int64_t N, int64_t K, int num_sms, int smem_optin, TcPlan* pl)
{
    constexpr bool kFused = MODE != kModeBF16;
    const int64_t wtiles = (N + 127) / 128;
    const int64_t nk = (K + 63) / 64;
    int bn, num_acc = 2, splits = 1;
    int64_t dp_tiles = 0;
    if (!kFused) {
        bn = choose_bn(M, N, num_sms, 256, 32);
    } else {
        // The fused kernel's cost per k-block of a unit is nearly independent of
        // the token tile width (the dequantization of the weight tile and the
        // hand-offs dominate, about 0.55 us on B200), so wide tiles are preferred
        // and the SMs are filled by splitting K.  Joint search over the tile width
        // (two TMEM accumulators up to 192 tokens, one at 256, whose epilogue does
        // not overlap the next tile: weight 1.12) and the K split, in k-block units.
        // Two forms of split: every tile split sp ways, or whole tiles for the
        // whole rounds of the grid and only the remaining tiles split (sp x their
        // count <= one round), so that they fill the last round instead of leaving
        // most SMs idle in it.
        //   cost = rounds x (k-blocks per unit + 4) x w
        //        + [split] (4 + fp32 partial traffic 8 x sp x split tiles x bn x 128 bytes at HBM speed)
        // The second form's cost carries 5% more: a last round that leaves most
        // SMs idle runs faster per tile than a full one, which the rounds count
        // does not see (on B200 it paid at 512 and 2048 tokens of the 12288 x 4096
        // projection, predicted 12% and 9% cheaper, and not at 4096, predicted 3%).
        // Ties go to the wider tile, then to the form found first.
        double best = 1e300;
        bn = 16;
        const int64_t maxb = std::min<int64_t>(256, (M + 15) / 16 * 16);
        auto consider = [&](double c, int b, int acc, int sp, int64_t dp) {
            if (c < best - 1e-9 || (c < best + 1e-9 && b > bn)) {
                best = c;
                bn = b;
                num_acc = acc;
                splits = sp;
                dp_tiles = dp;
            }
        };
        for (int b = 16; b <= maxb; b += 16) {
            if (b > 192 && b < maxb && b != 256) continue;      // one accumulator: only the widest tile
            const int acc = b > 192 ? 1 : 2;
            const double w = acc == 1 ? 1.12 : 1.0;
            const int64_t tiles = ((M + b - 1) / b) * wtiles;
            const double tile_elems = (double)b * 128.0;
            for (int sp = 1; sp <= 8; ++sp) {                   // every tile split sp ways
                if (sp > 1 && nk / sp < 4) break;
                const int64_t rounds = (tiles * sp + num_sms - 1) / num_sms;
                const double reduce = sp > 1 ? 4.0 + (double)sp * (double)tiles * tile_elems * 2.24e-6 : 0.0;
                consider((double)rounds * (double)((nk + sp - 1) / sp + 4) * w + reduce, b, acc, sp,
                         sp > 1 ? 0 : tiles);
            }
            const int64_t dp = tiles / num_sms * num_sms, tail = tiles - dp;
            for (int sp = 2; dp > 0 && tail > 0 && sp <= 8 && tail * sp <= num_sms; ++sp) {   // only the tail split
                if (nk / sp < 4) break;
                const double c = (double)(dp / num_sms) * (double)(nk + 4) * w + (double)((nk + sp - 1) / sp + 4) * w +
                                 4.0 + (double)sp * (double)tail * tile_elems * 2.24e-6;
                consider(c * 1.05, b, acc, sp, dp);
            }
        }
    }
    const int acc_stride = kFused ? (bn + 31) / 32 * 32 : 256;
    const uint32_t stage = tc_stage_bytes(MODE, bn);
    const int budget = smem_optin - 1024 - 512;
    int stages = std::min<int>(8, budget / (int)stage);
    if (kFused) stages = std::min(stages, (512 - num_acc * acc_stride) / 32);
    if (stages < 3) return false;
    pl->bn = bn;
    pl->num_acc = num_acc;
    pl->acc_stride = acc_stride;
    pl->stages = stages;
    pl->tiles = ((M + bn - 1) / bn) * wtiles;
    pl->splits = splits;
    pl->dp_tiles = splits > 1 ? dp_tiles : pl->tiles;
    pl->ws_bytes = splitk_ws_bytes(splits, pl->tiles - pl->dp_tiles, bn);
    return true;
}

// y = bf16(sum over splits of the partials) for the split tiles, in split order
// (deterministic).  Partials: [split][split tile][token of the tile][weight row of
// the tile]; one thread per 4 rows of one token (16-byte loads; 8-byte stores
// when N % 4 == 0 -- y and ws are 16-byte aligned).
__global__ void splitk_reduce_kernel(const float* __restrict__ ws, uint16_t* __restrict__ y, int M, int N, int bn,
                                     int m_tiles, int dp_tiles, int split_tiles, int splits)
{
    const int64_t per_tile = (int64_t)bn * 32;                       // 4-row groups per tile
    const int64_t total = (int64_t)split_tiles * per_tile;
    const int64_t split_stride = (int64_t)split_tiles * bn * 128;   // floats
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        const int j = (int)(i / per_tile);
        const int e = (int)(i - (int64_t)j * per_tile);
        const int m = e >> 5, r4 = (e & 31) * 4;
        const int t = dp_tiles + j;
        const int tok = (t % m_tiles) * bn + m, row = (t / m_tiles) * 128 + r4;
        if (tok >= M || row >= N) continue;
        const float* src = ws + ((int64_t)j * bn + m) * 128 + r4;
        float4 a = *reinterpret_cast<const float4*>(src);
        for (int sp = 1; sp < splits; ++sp) {
            const float4 b = *reinterpret_cast<const float4*>(src + sp * split_stride);
            a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
        }
        uint16_t* dst = y + (int64_t)tok * N + row;
        if ((N & 3) == 0) {                                          // then row + 4 <= N
            *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16x2_rn(a.x, a.y), pack_bf16x2_rn(a.z, a.w));
        } else {
            const float v[4] = {a.x, a.y, a.z, a.w};
            for (int k = 0; k < 4 && row + k < N; ++k) dst[k] = (uint16_t)f32_to_bf16_bits(v[k]);
        }
    }
}

template <int MODE>
bq_status launch_tc(const DeviceInfo& di, int dev, const uint16_t* x, const void* a_src, const uint16_t* scales,
                    const uint16_t* biases, uint16_t* y, int64_t M, int64_t N, int64_t K, cudaStream_t st,
                    void* ws = nullptr, size_t ws_bytes = 0, int group_size = 64)
{
    using C = TcCfg<MODE>;
    if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX) return BQ_ERR_SHAPE;
    TcPlan pl;
    if (!plan_tc<MODE>(M, N, K, di.num_sms, di.max_smem_optin, &pl)) return BQ_ERR_UNSUPPORTED;
    // K splits only with a workspace that holds their partial sums
    if (pl.splits > 1 && (!ws || ws_bytes < pl.ws_bytes)) {
        pl.splits = 1;
        pl.dp_tiles = pl.tiles;
    }
    const int bn = pl.bn, stages = pl.stages;
    const uint32_t stage = tc_stage_bytes(MODE, bn);
    // one CTA per SM: the kernel allocates all 512 TMEM columns
    const size_t smem = std::max<size_t>(1024 + (size_t)stages * stage + 512, (size_t)di.max_smem_optin / 2 + 1024);

    CUtensorMap tm_x, tm_a;
    if (!make_map(&tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, M, K, bn, 64, CU_TENSOR_MAP_SWIZZLE_128B))
        return BQ_ERR_CUDA;
    bool ok;
    if (MODE == kModeBF16)
        ok = make_map(&tm_a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a_src, N, K, 128, 64, CU_TENSOR_MAP_SWIZZLE_128B);
    else
        ok = make_map(&tm_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a_src, N, (MODE == kModeAff8) ? K : K / 2, 128,
                      C::kCodeBytesPerRow, CU_TENSOR_MAP_SWIZZLE_NONE);   // packed code bytes per row
    if (!ok) return BQ_ERR_CUDA;

    static bool attr_done[kMaxDevices] = {};
    if (!attr_done[dev]) {
        if (cudaFuncSetAttribute(tc_gemm_kernel<MODE, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 di.max_smem_optin) != cudaSuccess ||
            (MODE != kModeBF16 && cudaFuncSetAttribute(tc_gemm_kernel<MODE, MODE != kModeBF16>,
                                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                       di.max_smem_optin) != cudaSuccess))
            return BQ_ERR_CUDA;
        attr_done[dev] = true;
    }
    TcParams p;
    p.scales = scales;
    p.biases = biases;
    p.y = y;
    p.M = (int)M;
    p.N = (int)N;
    p.K = (int)K;
    p.bn = bn;
    p.stages = stages;
    p.m_tiles = (int)((M + bn - 1) / bn);
    const int64_t tiles = (int64_t)p.m_tiles * ((N + 127) / 128);
    if (tiles > INT32_MAX) return BQ_ERR_SHAPE;
    p.tiles = (int)tiles;
    p.acc_stride = pl.acc_stride;
    p.num_acc = pl.num_acc;
    p.splits = pl.splits;
    p.dp_tiles = (int)pl.dp_tiles;
    p.ws = pl.splits > 1 ? reinterpret_cast<float*>(ws) : nullptr;
    {
        const int gs = (MODE == kModeQ4_0 || MODE == kModeBF16) ? 32 : group_size;
        p.gs_shift = gs == 32 ? 5 : gs == 64 ? 6 : 7;
        p.vec_scales = ((K >> p.gs_shift) % 8 == 0) ? 1 : 0;   // every row starts and ends on whole windows
    }
    const int64_t units = pl.dp_tiles + (tiles - pl.dp_tiles) * pl.splits;
    const unsigned grid = (unsigned)std::min<int64_t>(units, di.num_sms);
    if (MODE != kModeBF16 && pl.num_acc == 1)
        tc_gemm_kernel<MODE, MODE != kModeBF16><<<grid, C::kThreads, smem, st>>>(tm_x, tm_a, p);
    else
        tc_gemm_kernel<MODE, false><<<grid, C::kThreads, smem, st>>>(tm_x, tm_a, p);
    if (pl.splits > 1) {
        bq_status r = launch_status();
        if (r != BQ_OK) return r;
        const int64_t split_tiles = tiles - pl.dp_tiles;
        const int64_t groups = split_tiles * bn * 32;
        const unsigned rgrid = (unsigned)std::max<int64_t>(1, std::min<int64_t>((groups + 255) / 256, 4 * di.num_sms));
        splitk_reduce_kernel<<<rgrid, 256, 0, st>>>(p.ws, y, (int)M, (int)N, bn, p.m_tiles, p.dp_tiles,
                                                    (int)split_tiles, pl.splits);
    }
    return launch_status();
}

// ------------------------------------------------------------------ GEMV
template <Fmt F, int NT, int RT, int KS, int PIPE, int MINB>
bq_status launch_gemv_cfg(const uint16_t* x, const void* wq, const uint16_t* s, const uint16_t* b, uint16_t* y,
                          int64_t M, int64_t N, int64_t K, int group_size, cudaStream_t st)
{
    const int64_t rows_per_cta = 16 * RT;
    const int64_t grid = (N + rows_per_cta - 1) / rows_per_cta;
    if (grid > INT32_MAX) return BQ_ERR_SHAPE;
    gemv_kernel<F, NT, RT, KS, PIPE, MINB><<<(unsigned)grid, 32 * KS, 0, st>>>(
        x, reinterpret_cast<const uint8_t*>(wq), s, b, y, (int)M, (int)N, (int)K, group_size);
    return launch_status();
}

template <Fmt F>
bq_status launch_gemv(const uint16_t* x, const void* wq, const uint16_t* s, const uint16_t* b, uint16_t* y,
                      int64_t M, int64_t N, int64_t K, int group_size, cudaStream_t st)
{
    if (N > INT32_MAX || K > INT32_MAX) return BQ_ERR_SHAPE;
    // Launch shapes measured on B200 at N = 12288, K = 4096: 32 weight rows per CTA,
    // K split over 4 (8 at M > 16) warps, 2-deep load pipeline; MINB CTAs per SM
    // keep the whole grid resident in one wave.
    if (M <= 8) return launch_gemv_cfg<F, 1, 2, 8, 1, 2>(x, wq, s, b, y, M, N, K, group_size, st);
    if (M <= 16) return launch_gemv_cfg<F, 2, 2, 4, 2, 2>(x, wq, s, b, y, M, N, K, group_size, st);
    return launch_gemv_cfg<F, 4, 2, 8, 1, 1>(x, wq, s, b, y, M, N, K, group_size, st);
}

bq_status library_workspace(int dev, cudaStream_t st, size_t need, void** out);

// ------------------------------------------------------------------ streamed decode GEMV
// Plan of gemv_stream_kernel for one problem: K chunk, ring depth, grid, the
// shared-memory carve-up and the activation tables.  Applies to one or two
// tokens, Q4_0 and affine 4/8-bit, when K is a multiple of 8 groups (every
// row's codes and scales of a chunk are then whole 16-byte runs that 16-byte
// copies can move); false otherwise.
constexpr int kSgWarps = 8;
constexpr int kSgStaticSmem = 1024;   // the kernel's static shared arrays, rounded up

struct SgPlan {
    SGemvParams prm{};
    int grid = 0;
    int su = 0;               // units of every warp's slice of a full chunk when equal and 8/16/32, else 0
    size_t smem = 0;
    int prep_grid = 0;        // CTAs of gemv_int_prep_kernel
    size_t tab_bytes = 0;     // device bytes of its tables and flags
};

// The matrices of one streamed launch: one, or up to kSgMaxMats sharing x.
struct SgMats {
    int count = 0;
    const void* wq[kSgMaxMats] = {};
    const uint16_t* scales[kSgMaxMats] = {};
    const uint16_t* biases[kSgMaxMats] = {};
    uint16_t* y[kSgMaxMats] = {};
    int64_t N[kSgMaxMats] = {};
};

// Activation-table bytes of the streamed GEMV (slices, group table, one flag
// word per prep CTA), or 0 when it does not apply to (fmt, M, K).
size_t stream_gemv_table_bytes(WFmt fmt, int group_size, int64_t M, int64_t K, int* prep_grid = nullptr)
{
    if (fmt != WFmt::Q4_0 && fmt != WFmt::AFF4 && fmt != WFmt::AFF8) return 0;
    const int gs = fmt == WFmt::Q4_0 ? 32 : group_size;
    if (M < 1 || M > kSgIntTokens || K < 1 || K > INT32_MAX / 16 || K % (8 * gs) != 0) return 0;
    const int64_t items = M * (K / 32) * 4;
    const int64_t grid = (items + kSgPrepThreads - 1) / kSgPrepThreads;
    if (prep_grid) *prep_grid = (int)grid;
    return (size_t)((K / 32) * kSgIntStepBytes + (K / gs) * kSgIntCtabBytes + (grid * 4 + 15) / 16 * 16);
}

// BQ_PATH_GEMV takes the streamed kernel where it measured faster than the
// register-streaming one on B200 (N = 12288, K = 4096, graph-timed launches
// over rotating weight copies, TMA-fed variant): one token (Q4_0 10.85 against
// 12.58 us, affine 4-bit 10.28 / 13.26, affine 8-bit 12.44 / 18.3) and two
// (12.30 / 12.60, 11.74 / 13.38, 13.79 / 18.3).
// It runs one CTA per SM and pays a fixed start per CTA (its activation slices,
// the ring's fill), so it needs several 16-row tiles per SM: with the Llama-3.2-1B
// stack's matrices (32 to 1024 tiles, K = 2048 or 8192) one token took 549 against
// 441 us per stack.  It is taken where it was measured faster: K >= 4096 and at
// least 4 tiles per SM.
bool stream_gemv_preferred(WFmt fmt, int64_t M, int64_t ntiles, int64_t K, int num_sms)
{
    (void)fmt;
    if (K < 4096 || ntiles < 4 * (int64_t)num_sms) return false;
    return M <= kSgIntTokens;
}

bool plan_stream_gemv(WFmt fmt, int group_size, int64_t M, const SgMats& mats, int64_t K, const DeviceInfo& di,
                      SgPlan* pl)
{
    int prep_grid = 0;
    const size_t tab_bytes = stream_gemv_table_bytes(fmt, group_size, M, K, &prep_grid);
    if (tab_bytes == 0 || mats.count < 1 || mats.count > kSgMaxMats) return false;
    const int gs = fmt == WFmt::Q4_0 ? 32 : group_size;
    const int bits = fmt == WFmt::AFF8 ? 8 : 4, E = bits == 8 ? 16 : 32;
    const int upg = gs / E, atom_units = upg > 2 ? upg : 2;
    // K chunk: whole rows up to 4096 elements (a multiple of 8 x 128); 8-bit codes in
    // 2048-element chunks measured slower (21.4 against 17.4 us at N = 12288, K = 4096)
    const int kc = (int)std::min<int64_t>(K, 4096);
    const int nchunks = (int)((K + kc - 1) / kc);
    SGemvParams& p = pl->prm;
    p = SGemvParams{};
    int64_t ntiles = 0;
    p.count = mats.count;
    for (int i = 0; i < mats.count; ++i) {
        if (mats.N[i] < 0 || mats.N[i] > INT32_MAX / 2) return false;
        p.tile_begin[i] = (int)ntiles;
        ntiles += (mats.N[i] + 15) / 16;
        if (ntiles > INT32_MAX / 2) return false;
        p.wq[i] = reinterpret_cast<const uint8_t*>(mats.wq[i]);
        p.scales[i] = mats.scales[i];
        p.biases[i] = mats.biases[i];
        p.y[i] = mats.y[i];
        p.N[i] = (int)mats.N[i];
    }
    p.tile_begin[mats.count] = (int)ntiles;
    if (ntiles == 0) return false;
    // one CTA per SM over a contiguous range of tiles; at most 8 tiles per CTA
    // (more CTAs, in waves, for very tall W)
    const int64_t grid = ntiles <= 8 * (int64_t)di.num_sms ? std::min<int64_t>(ntiles, di.num_sms) : (ntiles + 7) / 8;
    const int64_t tcap = (ntiles + grid - 1) / grid;
    // a warp's slice of a full chunk: at most ceil(atoms / warps) atoms; its scale
    // run covers 2 bytes per group plus up to 15 bytes of alignment on each side
    const int64_t natoms = kc / E / atom_units;
    const int64_t nc_max = (natoms + kSgWarps - 1) / kSgWarps * atom_units;       // 16-byte code units
    const int64_t gpw = nc_max / upg;                                              // groups
    const int64_t ns_max = (2 * gpw + 30) / 16;                                    // 16-byte scale runs
    // row pitches: odd multiples of 16 bytes, so 8 rows fall in 8 distinct bank groups
    auto odd16 = [](int64_t units) { return (units % 2 == 0 ? units + 1 : units) * 16; };
    const int64_t code_pitch = odd16(nc_max + 1), scale_pitch = odd16(ns_max);
    const bool affine = fmt != WFmt::Q4_0;
    const int64_t wstage = 16 * code_pitch + 16 * scale_pitch * (affine ? 2 : 1);
    // shared memory: the activation tables ([K/32 steps] x 256 bytes, [groups] x
    // 64 bytes), the per-warp partial sums of the CTA's tiles, the rings
    const int64_t x_bytes = (K / 32) * kSgIntStepBytes, c_bytes = (K / gs) * kSgIntCtabBytes;
    int64_t off = 0;
    const int64_t off_x = off;
    off = (off + x_bytes + 127) / 128 * 128;
    const int64_t off_c = off;
    off = (off + c_bytes + 127) / 128 * 128;
    const int64_t red_cols = 2;
    const int64_t off_red = off;
    off = (off + tcap * kSgWarps * 16 * red_cols * 4 + 127) / 128 * 128;
    const int64_t off_ring = off;
    const int64_t budget = (int64_t)di.max_smem_optin - kSgStaticSmem;
    const int64_t stages = std::min<int64_t>(4, (budget - off_ring) / (kSgWarps * wstage));
    if (stages < 2) return false;
    p.M = (int)M;
    p.K = (int)K;
    p.kc = kc;
    p.nchunks = nchunks;
    p.ntiles = (int)ntiles;
    p.stages = (int)stages;
    p.code_pitch = (uint32_t)code_pitch;
    p.scale_pitch = (uint32_t)scale_pitch;
    p.wstage_bytes = (uint32_t)wstage;
    p.red_cols = (int)red_cols;
    p.off_x = (uint32_t)off_x;
    p.off_c = (uint32_t)off_c;
    p.off_red = (uint32_t)off_red;
    p.off_ring = (uint32_t)off_ring;
    p.tab_c_off = (uint32_t)x_bytes;
    p.tab_f_off = (uint32_t)(x_bytes + c_bytes);
    p.nflags = prep_grid;
    pl->grid = (int)grid;
    pl->prep_grid = prep_grid;
    pl->tab_bytes = tab_bytes;
    const int64_t su = natoms % kSgWarps == 0 ? natoms / kSgWarps * atom_units : 0;
    pl->su = (su == 8 || su == 16 || su == 32) ? (int)su : 0;
    pl->smem = (size_t)(off_ring + stages * kSgWarps * wstage);
    return true;
}

// Launch with programmatic stream serialization: the kernel's launch and
// prologue may overlap the previous kernel on the stream; its reads of x,
// tables, W and scales and its writes come after griddepcontrol.wait.
template <typename KernelT, typename... Args>
bq_status launch_pdl(KernelT kern, int grid, int threads, size_t smem, cudaStream_t st, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3((unsigned)threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, args...) != cudaSuccess) {
        cudaGetLastError();
        return BQ_ERR_CUDA;
    }
    return launch_status();
}

template <Fmt F, int GS, int SU>
bq_status launch_stream_gemv_su(SgPlan& pl, int dev, const DeviceInfo& di, cudaStream_t st)
{
    auto kern = gemv_stream_kernel<F, GS, kSgWarps, SU>;
    static bool attr_done[kMaxDevices] = {};
    if (!attr_done[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 di.max_smem_optin - kSgStaticSmem) != cudaSuccess)
            return BQ_ERR_CUDA;
        attr_done[dev] = true;
    }
    return launch_pdl(kern, pl.grid, 32 * kSgWarps, pl.smem, st, pl.prm);
}

// The activation tables, then the streamed kernel.
template <Fmt F, int GS>
bq_status launch_stream_gemv(SgPlan& pl, int dev, const DeviceInfo& di, const uint16_t* x, uint8_t* tab,
                             cudaStream_t st)
{
    pl.prm.x = x;
    pl.prm.tab = tab;
    bq_status s = launch_pdl(gemv_int_prep_kernel<F, GS>, pl.prep_grid, kSgPrepThreads, 0, st, x, pl.prm.M,
                             pl.prm.K, tab, pl.prm.tab_c_off, pl.prm.tab_f_off);
    if (s != BQ_OK) return s;
    switch (pl.su) {
    case 8: return launch_stream_gemv_su<F, GS, 8>(pl, dev, di, st);
    case 16: return launch_stream_gemv_su<F, GS, 16>(pl, dev, di, st);
    case 32: return launch_stream_gemv_su<F, GS, 32>(pl, dev, di, st);
    default: return launch_stream_gemv_su<F, GS, 0>(pl, dev, di, st);
    }
}

// Plan of the TMA-fed kernel: stages of CH = 16 (else 8) 128-byte code chunks
// per row, whole rows split into nchunks stages; false when K does not split
// that way or a stage's scales are not whole 16-byte rows.
struct SgTmaPlan {
    STmaParams prm{};
    int grid = 0, ch = 0;
    size_t smem = 0;
};

// The TMA kernel's stage shape and shared-memory carve-up for (fmt, M, K) and
// ntiles 16-row tiles on a device with num_sms SMs and smem_optin bytes of
// shared memory per block; false when it does not apply.
struct SgTmaShape {
    int ch = 0, stages = 0, nchunks = 0, grid = 0;
    int64_t stage_elems = 0, stage_groups = 0, scale_row = 0, stage_pitch = 0;
    int64_t off_x = 0, off_c = 0, off_red = 0, off_bar = 0, off_raw = 0, off_stage = 0, smem = 0;
};

bool tma_shape(WFmt fmt, int group_size, int64_t M, int64_t ntiles, int64_t K, int num_sms, int smem_optin,
               SgTmaShape* sh)
{
    if (stream_gemv_table_bytes(fmt, group_size, M, K) == 0 || ntiles < 1) return false;
    const int gs = fmt == WFmt::Q4_0 ? 32 : group_size;
    const int bits = fmt == WFmt::AFF8 ? 8 : 4, E = bits == 8 ? 16 : 32;
    const int upg = gs / E, atom_units = upg > 2 ? upg : 2;
    const int64_t row_bytes = K * bits / 8;
    if (row_bytes % 128 != 0) return false;
    const int64_t row_chunks = row_bytes / 128;
    const int ch = row_chunks % 16 == 0 ? 16 : row_chunks % 8 == 0 ? 8 : 0;
    if (ch == 0 || ch % atom_units != 0) return false;
    SgTmaShape& h = *sh;
    h.ch = ch;
    h.stage_elems = (int64_t)ch * 128 * 8 / bits;
    h.stage_groups = h.stage_elems / gs;
    h.scale_row = h.stage_groups * 2;
    if (h.scale_row % 16 != 0) return false;
    h.nchunks = (int)(row_chunks / ch);
    h.grid = (int)(ntiles <= 8 * (int64_t)num_sms ? std::min<int64_t>(ntiles, num_sms) : (ntiles + 7) / 8);
    const int64_t tcap = (ntiles + h.grid - 1) / h.grid;
    const bool affine = fmt != WFmt::Q4_0;
    auto up = [](int64_t v, int64_t a) { return (v + a - 1) / a * a; };
    h.stage_pitch = up((int64_t)ch * 2048 + 16 * h.scale_row * (affine ? 2 : 1), 1024);
    int64_t off = 0;
    h.off_x = off;
    off = up(off + (K / 32) * kSgIntStepBytes, 128);
    h.off_c = off;
    off = up(off + (K / gs) * kSgIntCtabBytes, 128);
    h.off_red = off;
    off = up(off + tcap * kSgWarpsTma * 16 * M * 4, 128);           // one column per token
    h.off_bar = off;
    off = up(off + (2 * kSgMaxStagesTma + 1) * 8, 128);
    h.off_raw = off;                                                 // x itself, bf16 [M][K]
    off = up(off + M * K * 2, 1024);
    h.off_stage = off;
    const int64_t budget = (int64_t)smem_optin - 1024;               // 1 KB to align the base
    // as many stages as fit, up to 4 (5 measured slower for the 4-bit formats: 13.2
    // against 12.7 us for Q4_0 at M = 1)
    h.stages = (int)std::min<int64_t>(kSgMaxStagesTma, (budget - off) / h.stage_pitch);
    if (h.stages < 2) return false;
    h.smem = off + h.stages * h.stage_pitch + 1024;
    return true;
}

bool plan_stream_gemv_tma(WFmt fmt, int group_size, int64_t M, const SgMats& mats, int64_t K, const DeviceInfo& di,
                          SgTmaPlan* pl)
{
    if (mats.count < 1 || mats.count > kSgMaxMats) return false;
    int64_t nt_all = 0;
    for (int i = 0; i < mats.count; ++i) nt_all += (std::max<int64_t>(mats.N[i], 0) + 15) / 16;
    SgTmaShape h;
    if (!tma_shape(fmt, group_size, M, nt_all, K, di.num_sms, di.max_smem_optin, &h)) return false;
    const int gs = fmt == WFmt::Q4_0 ? 32 : group_size;
    const int bits = fmt == WFmt::AFF8 ? 8 : 4;
    const int64_t row_bytes = K * bits / 8;
    const int ch = h.ch;
    const int64_t stage_groups = h.stage_groups;
    SgTmaPlan& P = *pl;
    STmaParams& q = P.prm;
    q = STmaParams{};
    SGemvParams& p = q.g;
    int64_t ntiles = 0;
    p.count = mats.count;
    for (int i = 0; i < mats.count; ++i) {
        if (mats.N[i] < 0 || mats.N[i] > INT32_MAX / 2) return false;
        p.tile_begin[i] = (int)ntiles;
        ntiles += (mats.N[i] + 15) / 16;
        if (ntiles > INT32_MAX / 2) return false;
        p.wq[i] = reinterpret_cast<const uint8_t*>(mats.wq[i]);
        p.scales[i] = mats.scales[i];
        p.biases[i] = mats.biases[i];
        p.y[i] = mats.y[i];
        p.N[i] = (int)mats.N[i];
        if (mats.N[i] == 0) continue;
        if (!make_code_map_3d(&q.codes[i], mats.wq[i], mats.N[i], row_bytes, ch)) return false;
        if (!make_scale_map_3d(&q.scales[i], mats.scales[i], mats.N[i], K / gs, (int)(stage_groups / 8)))
            return false;
        if (fmt != WFmt::Q4_0 &&
            !make_scale_map_3d(&q.biases[i], mats.biases[i], mats.N[i], K / gs, (int)(stage_groups / 8)))
            return false;
    }
    p.tile_begin[mats.count] = (int)ntiles;
    if (ntiles == 0) return false;
    const bool affine = fmt != WFmt::Q4_0;
    p.M = (int)M;
    p.K = (int)K;
    p.kc = (int)h.stage_elems;
    p.nchunks = h.nchunks;
    p.ntiles = (int)ntiles;
    p.stages = h.stages;
    p.red_cols = (int)M;
    p.off_x = (uint32_t)h.off_x;
    p.off_c = (uint32_t)h.off_c;
    p.off_red = (uint32_t)h.off_red;
    q.off_stage = (uint32_t)h.off_stage;
    q.off_raw = (uint32_t)h.off_raw;
    q.stage_pitch = (uint32_t)h.stage_pitch;
    q.scale_row_bytes = (uint32_t)h.scale_row;
    q.stage_tx = (uint32_t)(ch * 2048 + 16 * h.scale_row * (affine ? 2 : 1));
    q.off_bar = (uint32_t)h.off_bar;
    P.grid = h.grid;
    P.ch = ch;
    P.smem = (size_t)h.smem;
    return true;
}

template <Fmt F, int GS, int CH>
bq_status launch_stream_gemv_tma_ch(SgTmaPlan& pl, int dev, const DeviceInfo& di, cudaStream_t st)
{
    auto kern = gemv_tma_kernel<F, GS, CH>;
    static bool attr_done[kMaxDevices] = {};
    if (!attr_done[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, di.max_smem_optin) !=
            cudaSuccess)
            return BQ_ERR_CUDA;
        attr_done[dev] = true;
    }
    return launch_pdl(kern, pl.grid, 32 * (kSgWarpsTma + 1), pl.smem, st, pl.prm);
}

// One launch: the kernel builds its activation tables itself.
template <Fmt F, int GS>
bq_status launch_stream_gemv_tma(SgTmaPlan& pl, int dev, const DeviceInfo& di, const uint16_t* x, cudaStream_t st)
{
    pl.prm.g.x = x;
    pl.prm.g.tab = nullptr;
    return pl.ch == 16 ? launch_stream_gemv_tma_ch<F, GS, 16>(pl, dev, di, st)
                       : launch_stream_gemv_tma_ch<F, GS, 8>(pl, dev, di, st);
}

// The streamed kernel when its plan applies (returns true and the launch status
// in *out), else false and the caller takes the register-streaming GEMV.  The
// TMA-fed variant runs where its stages fit K, the cp.async one otherwise.  Its
// tables go in the caller's workspace when one is given (false if it is too
// small), else in the library's buffer of this stream.
std::mutex g_sg_mu;                        // the TMA plan's static storage

bool try_stream_gemv(WFmt fmt, int group_size, const uint16_t* x, const SgMats& mats, int64_t M, int64_t K, int dev,
                     const DeviceInfo& di, cudaStream_t st, void* workspace, size_t workspace_bytes, bq_status* out)
{
    static SgTmaPlan tp;                   // large (tensor maps): not on the stack
    std::lock_guard<std::mutex> lk(g_sg_mu);
    if (plan_stream_gemv_tma(fmt, group_size, M, mats, K, di, &tp)) {     // needs no device scratch
        switch (fmt) {
        case WFmt::Q4_0: *out = launch_stream_gemv_tma<Fmt::Q4_0, 32>(tp, dev, di, x, st); break;
        case WFmt::AFF4:
            *out = group_size == 32   ? launch_stream_gemv_tma<Fmt::AFF4, 32>(tp, dev, di, x, st)
                   : group_size == 64 ? launch_stream_gemv_tma<Fmt::AFF4, 64>(tp, dev, di, x, st)
                                      : launch_stream_gemv_tma<Fmt::AFF4, 128>(tp, dev, di, x, st);
            break;
        default:
            *out = group_size == 32   ? launch_stream_gemv_tma<Fmt::AFF8, 32>(tp, dev, di, x, st)
                   : group_size == 64 ? launch_stream_gemv_tma<Fmt::AFF8, 64>(tp, dev, di, x, st)
                                      : launch_stream_gemv_tma<Fmt::AFF8, 128>(tp, dev, di, x, st);
            break;
        }
        return true;
    }
    SgPlan pl;
    if (!plan_stream_gemv(fmt, group_size, M, mats, K, di, &pl)) return false;
    void* tab = workspace;
    if (tab) {
        if (workspace_bytes < pl.tab_bytes) return false;
    } else if ((*out = library_workspace(dev, st, pl.tab_bytes, &tab)) != BQ_OK) {
        return true;
    }
    uint8_t* t = reinterpret_cast<uint8_t*>(tab);
    switch (fmt) {
    case WFmt::Q4_0: *out = launch_stream_gemv<Fmt::Q4_0, 32>(pl, dev, di, x, t, st); break;
    case WFmt::AFF4:
        *out = group_size == 32   ? launch_stream_gemv<Fmt::AFF4, 32>(pl, dev, di, x, t, st)
               : group_size == 64 ? launch_stream_gemv<Fmt::AFF4, 64>(pl, dev, di, x, t, st)
                                  : launch_stream_gemv<Fmt::AFF4, 128>(pl, dev, di, x, t, st);
        break;
    default:
        *out = group_size == 32   ? launch_stream_gemv<Fmt::AFF8, 32>(pl, dev, di, x, t, st)
               : group_size == 64 ? launch_stream_gemv<Fmt::AFF8, 64>(pl, dev, di, x, t, st)
                                  : launch_stream_gemv<Fmt::AFF8, 128>(pl, dev, di, x, t, st);
        break;
    }
    return true;
}

SgMats one_matrix(const void* wq, const uint16_t* s, const uint16_t* b, uint16_t* y, int64_t N)
{
    SgMats m;
    m.count = 1;
    m.wq[0] = wq;
    m.scales[0] = s;
    m.biases[0] = b;
    m.y[0] = y;
    m.N[0] = N;
    return m;
}

// Decode GEMV for affine weights of any width (2-, 3- and 6-bit use it): one
// launch per kGaMaxM tokens (each pass a contiguous block of x's and y's rows,
// reading W again), up to kGaForcedMaxM tokens.
bq_status launch_gemv_affine(WFmt fmt, const uint16_t* x, const void* wq, const uint16_t* s, const uint16_t* b,
                             uint16_t* y, int64_t M, int64_t N, int64_t K, int group_size, cudaStream_t st)
{
    if (N > INT32_MAX || K > INT32_MAX || M > kGaForcedMaxM) return BQ_ERR_SHAPE;
    if (M > kGaMaxM) {
        for (int64_t m0 = 0; m0 < M; m0 += kGaMaxM) {
            const bq_status r = launch_gemv_affine(fmt, x + m0 * K, wq, s, b, y + m0 * N,
                                                   std::min<int64_t>(kGaMaxM, M - m0), N, K, group_size, st);
            if (r != BQ_OK) return r;
        }
        return BQ_OK;
    }
    const int64_t rows_per_cta = (int64_t)kGaRows * kGaWarps;
    const unsigned grid = (unsigned)((N + rows_per_cta - 1) / rows_per_cta);
    const uint32_t* w = reinterpret_cast<const uint32_t*>(wq);
    auto go = [&](auto bits_tag, auto mt_tag) {
        constexpr int B = decltype(bits_tag)::value, MT = decltype(mt_tag)::value;
        gemv_affine_kernel<B, MT><<<grid, 32 * kGaWarps, 0, st>>>(x, w, s, b, y, (int)M, (int)N, (int)K, group_size);
    };
    auto by_m = [&](auto bits_tag) {
        if (M <= 1) go(bits_tag, std::integral_constant<int, 1>());
        else if (M <= 2) go(bits_tag, std::integral_constant<int, 2>());
        else if (M <= 4) go(bits_tag, std::integral_constant<int, 4>());
        else go(bits_tag, std::integral_constant<int, 8>());
    };
    switch (fmt) {
    case WFmt::AFF2: by_m(std::integral_constant<int, 2>()); break;
    case WFmt::AFF3: by_m(std::integral_constant<int, 3>()); break;
    case WFmt::AFF6: by_m(std::integral_constant<int, 6>()); break;
    default: return BQ_ERR_UNSUPPORTED;
    }
    return launch_status();
}

// Decode GEMV over [K][N] affine weights (transpose = 0), 2-, 4- or 8-bit: up to
// kGtMaxM tokens when forced, up to kGtAutoMaxM when the dispatcher chooses (the
// measured crossover with the unfused pair on B200: the GEMV is ahead at 1 to 4
// tokens, behind at 8).
constexpr int64_t kGtMaxM = 8;
constexpr int64_t kGtAutoMaxM = 4;

// CTAs per cluster along K: as many as fit on the GPU at once beside the other
// clusters (one wave), at most 8, with at least 32 rows of K per CTA.
int gemv_t_split(int64_t N, int64_t K, int cols, int resident)
{
    const int64_t ncb = (N + cols - 1) / cols;
    int64_t ks = std::min<int64_t>(kGtMaxSplit, std::max<int64_t>(1, (int64_t)resident / ncb));
    while (ks > 1 && K < 32 * ks) --ks;
    return (int)ks;
}

template <int BITS, int MT>
bq_status launch_gemv_t_cfg(const uint16_t* x, const uint32_t* w, const uint16_t* s, const uint16_t* b, uint16_t* y,
                            int64_t M, int64_t N, int64_t K, int group_size, const DeviceInfo& di, cudaStream_t st)
{
    constexpr int U = MT == 1 && BITS != 8 ? 8 : 4;   // rows per batch (two batches in registers)
    constexpr int cols = 32 * gemv_t_cpl<MT>();
    auto kern = gemv_t_kernel<BITS, MT, U, 2>;
    static int per_sm = 0;                    // resident CTAs per SM (the same on every B200)
    if (per_sm == 0) {
        int v = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, kern, 32 * kGtWarps, 0) != cudaSuccess) {
            cudaGetLastError();
            v = 1;
        }
        per_sm = std::max(v, 1);
    }
    const int ks = gemv_t_split(N, K, cols, per_sm * di.num_sms);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((N + cols - 1) / cols), (unsigned)ks);
    cfg.blockDim = dim3(32 * kGtWarps);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = (unsigned)ks;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, x, w, s, b, y, (int)M, (int)N, (int)K, group_size) != cudaSuccess) {
        cudaGetLastError();
        return BQ_ERR_CUDA;
    }
    return launch_status();
}

bq_status launch_gemv_t(WFmt fmt, const uint16_t* x, const void* wq, const uint16_t* s, const uint16_t* b,
                        uint16_t* y, int64_t M, int64_t N, int64_t K, int group_size, const DeviceInfo& di,
                        cudaStream_t st)
{
    // the kernel indexes columns in int, up to one cluster's width past N
    if (N > INT32_MAX - 1024 || K > INT32_MAX || M > kGtMaxM) return BQ_ERR_SHAPE;
    const uint32_t* w = reinterpret_cast<const uint32_t*>(wq);
    auto by_m = [&](auto bits_tag) {
        constexpr int B = decltype(bits_tag)::value;
        if (M <= 1) return launch_gemv_t_cfg<B, 1>(x, w, s, b, y, M, N, K, group_size, di, st);
        if (M <= 2) return launch_gemv_t_cfg<B, 2>(x, w, s, b, y, M, N, K, group_size, di, st);
        if (M <= 4) return launch_gemv_t_cfg<B, 4>(x, w, s, b, y, M, N, K, group_size, di, st);
        return launch_gemv_t_cfg<B, 8>(x, w, s, b, y, M, N, K, group_size, di, st);
    };
    switch (fmt) {
    case WFmt::AFF2: return by_m(std::integral_constant<int, 2>());
    case WFmt::AFF4: return by_m(std::integral_constant<int, 4>());
    case WFmt::AFF8: return by_m(std::integral_constant<int, 8>());
    default: return BQ_ERR_UNSUPPORTED;
    }
}

template <Fmt F, int NT, int RT, int KS, int PIPE, int MINB>
bq_status launch_gemv_multi_cfg(const uint16_t* x, GemvMultiTable& tab, int64_t M, int64_t K, int group_size,
                                cudaStream_t st)
{
    tab.tile_begin[0] = 0;
    for (int i = 0; i < tab.count; ++i) {
        const int64_t end = tab.tile_begin[i] + ((int64_t)tab.N[i] + 16 * RT - 1) / (16 * RT);
        if (end > INT32_MAX) return BQ_ERR_SHAPE;
        tab.tile_begin[i + 1] = (int)end;
    }
    const int grid = tab.tile_begin[tab.count];
    if (grid == 0) return BQ_OK;
    gemv_multi_kernel<F, NT, RT, KS, PIPE, MINB><<<(unsigned)grid, 32 * KS, 0, st>>>(x, tab, (int)M, (int)K,
                                                                                  group_size);
    return launch_status();
}

// Same launch shapes as launch_gemv, all matrices in one grid.
template <Fmt F>
bq_status launch_gemv_multi(const uint16_t* x, GemvMultiTable& tab, int64_t M, int64_t K, int group_size,
                            cudaStream_t st)
{
    if (K > INT32_MAX) return BQ_ERR_SHAPE;
    if (M <= 8) return launch_gemv_multi_cfg<F, 1, 2, 8, 1, 2>(x, tab, M, K, group_size, st);
    if (M <= 16) return launch_gemv_multi_cfg<F, 2, 2, 4, 2, 2>(x, tab, M, K, group_size, st);
    return launch_gemv_multi_cfg<F, 4, 2, 8, 1, 1>(x, tab, M, K, group_size, st);
}

// ------------------------------------------------------------------ library workspace
// Scratch of the calls that get no caller workspace: one buffer per (device,
// stream), so calls on different streams never share one.  A buffer only grows
// (to the next power of two of the need), and a grown-out block is retired,
// not freed: CUDA graphs captured earlier keep pointing at valid memory.
// Retired blocks and live buffers are released when the process exits.
struct Workspace {
    void* ptr = nullptr;
    size_t bytes = 0;
};
struct WorkspaceKey {
    int dev;
    cudaStream_t stream;
    bool operator<(const WorkspaceKey& o) const { return dev != o.dev ? dev < o.dev : stream < o.stream; }
};
std::map<WorkspaceKey, Workspace> g_ws;
std::vector<void*> g_ws_retired;

bq_status library_workspace(int dev, cudaStream_t st, size_t need, void** out)
{
    std::lock_guard<std::mutex> lk(g_mu);
    Workspace& w = g_ws[WorkspaceKey{dev, st}];
    if (w.bytes < need) {
        size_t bytes = 1u << 20;
        while (bytes < need) bytes <<= 1;
        void* p = nullptr;
        if (cudaMalloc(&p, bytes) != cudaSuccess) {
            cudaGetLastError();
            return BQ_ERR_CUDA;
        }
        if (w.ptr) g_ws_retired.push_back(w.ptr);
        w.ptr = p;
        w.bytes = bytes;
    }
    *out = w.ptr;
    return BQ_OK;
}

// Workspace of a path: the bf16 copy of W for the pair; the K-split partial
// sums for the fused kernel when its plan splits K; the activation tables of
// the streamed decode GEMV (one or two tokens); 0 otherwise.
size_t workspace_for(int path, WFmt fmt, int group_size, int64_t M, int64_t N, int64_t K, int num_sms,
                     int smem_optin)
{
    if (path == BQ_PATH_DEQUANT_GEMM) return (size_t)N * (size_t)K * 2u;
    if ((path == BQ_PATH_GEMV && stream_gemv_preferred(fmt, M, (N + 15) / 16, K, num_sms)) ||
        path == BQ_PATH_GEMV_STREAM) {
        // the TMA-fed kernel builds its tables in shared memory; the cp.async one
        // takes them from device scratch
        if (!has_fast_paths(fmt)) return 0u;
        SgTmaShape h;
        if (tma_shape(fmt, group_size, M, (N + 15) / 16, K, num_sms, smem_optin, &h)) return 0u;
        return stream_gemv_table_bytes(fmt, group_size, M, K);
    }
    if (path == BQ_PATH_GEMV) return 0u;
    if (path != BQ_PATH_TC_FUSED || !has_fast_paths(fmt) || K % 64 != 0 || M > INT32_MAX || N > INT32_MAX ||
        K > INT32_MAX)
        return 0u;
    TcPlan pl;
    bool ok = fmt == WFmt::Q4_0  ? plan_tc<kModeQ4_0>(M, N, K, num_sms, smem_optin, &pl)
              : fmt == WFmt::AFF4 ? plan_tc<kModeAff4>(M, N, K, num_sms, smem_optin, &pl)
                                  : plan_tc<kModeAff8>(M, N, K, num_sms, smem_optin, &pl);
    return ok ? pl.ws_bytes : 0u;
}

bq_status dequant_any(WFmt fmt, const void* wq, const void* scales, const void* biases, uint16_t* out, int64_t N,
                      int64_t K, int group_size, const DeviceInfo& di, cudaStream_t st)
{
    if (fmt == WFmt::Q4_0) {
        const int64_t nb = N * (K / 32);
        q4_0_dequant_kernel<<<grid_for(nb, 256, di), 256, 0, st>>>(
            reinterpret_cast<const uint8_t*>(wq), reinterpret_cast<const uint16_t*>(scales), out, nb);
    } else {
        const uint32_t* w = reinterpret_cast<const uint32_t*>(wq);
        const uint16_t* sc = reinterpret_cast<const uint16_t*>(scales);
        const uint16_t* bi = reinterpret_cast<const uint16_t*>(biases);
        auto go = [&](auto bits_tag) {
            constexpr int B = decltype(bits_tag)::value;
            const int64_t nu = N * (K / AffUnit<B>::E);
            affine_dequant_kernel<B><<<grid_for(nu, 256, di), 256, 0, st>>>(w, sc, bi, out, nu, K, group_size);
        };
        switch (fmt) {
        case WFmt::AFF2: go(std::integral_constant<int, 2>()); break;
        case WFmt::AFF3: go(std::integral_constant<int, 3>()); break;
        case WFmt::AFF4: go(std::integral_constant<int, 4>()); break;
        case WFmt::AFF6: go(std::integral_constant<int, 6>()); break;
        default: go(std::integral_constant<int, 8>()); break;
        }
    }
    return launch_status();
}

// Affine W stored as R rows of C codes grouped along C, dequantized into its
// transpose out[C][R] (the weight operand of y = x . W for transpose = 0).
bq_status dequant_affine_t(WFmt fmt, const void* wq, const void* scales, const void* biases, uint16_t* out,
                           int64_t R, int64_t C, int group_size, const DeviceInfo& di, cudaStream_t st)
{
    const uint32_t* w = reinterpret_cast<const uint32_t*>(wq);
    const uint16_t* sc = reinterpret_cast<const uint16_t*>(scales);
    const uint16_t* bi = reinterpret_cast<const uint16_t*>(biases);
    const int64_t tiles = ((R + kTrRows - 1) / kTrRows) * ((C + kTrCols - 1) / kTrCols);
    const unsigned grid = (unsigned)std::max<int64_t>(1, std::min<int64_t>(tiles, (int64_t)di.num_sms * 8));
    auto go = [&](auto bits_tag) {
        constexpr int B = decltype(bits_tag)::value;
        affine_dequant_t_kernel<B><<<grid, 256, 0, st>>>(w, sc, bi, out, R, C, group_size);
    };
    switch (fmt) {
    case WFmt::AFF2: go(std::integral_constant<int, 2>()); break;
    case WFmt::AFF3: go(std::integral_constant<int, 3>()); break;
    case WFmt::AFF4: go(std::integral_constant<int, 4>()); break;
    case WFmt::AFF6: go(std::integral_constant<int, 6>()); break;
    default: go(std::integral_constant<int, 8>()); break;
    }
    return launch_status();
}

bq_status matmul_impl(const uint16_t* x, const void* wq, const void* scales, const void* biases, uint16_t* y,
                      int64_t M, int64_t N, int64_t K, int group_size, int bits, int transpose, int path,
                      void* workspace, size_t workspace_bytes, cudaStream_t st)
{
    if (transpose != 0 && transpose != 1) return BQ_ERR_UNSUPPORTED;
    if (path < BQ_PATH_AUTO || path > BQ_PATH_GEMV_STREAM) return BQ_ERR_UNSUPPORTED;
    if (M < 0 || N < 0 || K < 0) return BQ_ERR_SHAPE;
    // transpose = 0: y = x . W with W stored [K][N], codes and groups along N
    // (affine only: Q4_0 blocks run along K).  Up to kGtAutoMaxM tokens of 2-, 4-
    // or 8-bit codes (kGtMaxM when forced) run the decode GEMV over [K][N]
    // (gemv_t_kernel); otherwise the unfused pair with a transposing dequantize,
    // whose x rows must be 16-byte multiples.
    if (transpose == 0 && !biases) return BQ_ERR_UNSUPPORTED;
    WFmt fmt;
    bq_status s = transpose ? check_format(biases, N, K, group_size, bits, &fmt)
                            : check_format(biases, K, N, group_size, bits, &fmt);
    if (s != BQ_OK) return s;
    bool gemv_t = false;
    if (transpose == 0) {
        const bool gt_fmt = bits == 2 || bits == 4 || bits == 8;
        if (path == BQ_PATH_TC_FUSED || path == BQ_PATH_GEMV_STREAM || (path == BQ_PATH_GEMV && !(gt_fmt && M <= kGtMaxM)))
            return BQ_ERR_UNSUPPORTED;
        if (path == BQ_PATH_GEMV || (path == BQ_PATH_AUTO && gt_fmt && M <= kGtAutoMaxM)) {
            gemv_t = true;
            path = BQ_PATH_GEMV;
        } else {
            if (K % 8 != 0) return BQ_ERR_SHAPE;
            path = BQ_PATH_DEQUANT_GEMM;
        }
    }
    if (M == 0 || N == 0) return BQ_OK;      // empty problem: nothing is read or written
    int dev;
    DeviceInfo di;
    if (K == 0) {                            // empty sum: y = 0
        if (!y) return BQ_ERR_NULL;
        if (!aligned16(y)) return BQ_ERR_ALIGN;
        if ((s = current_device(&dev, &di)) != BQ_OK) return s;
        return cudaMemsetAsync(y, 0, (size_t)M * (size_t)N * 2u, st) == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
    }
    if (!x || !wq || !scales || !y) return BQ_ERR_NULL;
    if (!aligned16(x) || !aligned16(wq) || !aligned16(scales) || !aligned16(y) || (biases && !aligned16(biases)) ||
        (workspace && !aligned16(workspace)))
        return BQ_ERR_ALIGN;
    if (path == BQ_PATH_AUTO) path = select_path(M, K, fmt);
    if (!has_fast_paths(fmt) && (path == BQ_PATH_TC_FUSED || (path == BQ_PATH_GEMV && M > kGaForcedMaxM)))
        return BQ_ERR_UNSUPPORTED;
    if (path == BQ_PATH_GEMV && M > kGemvMaxM) return BQ_ERR_UNSUPPORTED;
    if (path == BQ_PATH_TC_FUSED && K % 64 != 0) return BQ_ERR_UNSUPPORTED;
    if (path == BQ_PATH_DEQUANT_GEMM && workspace && workspace_bytes < (size_t)N * (size_t)K * 2u)
        return BQ_ERR_WORKSPACE;

    if ((s = current_device(&dev, &di)) != BQ_OK) return s;
    const size_t need = workspace_for(path, fmt, group_size, M, N, K, di.num_sms, di.max_smem_optin);

    const uint16_t* sc = reinterpret_cast<const uint16_t*>(scales);
    const uint16_t* bi = reinterpret_cast<const uint16_t*>(biases);
    if (gemv_t) return launch_gemv_t(fmt, x, wq, sc, bi, y, M, N, K, group_size, di, st);
    switch (path) {
    case BQ_PATH_GEMV_STREAM:
        if (!has_fast_paths(fmt) || stream_gemv_table_bytes(fmt, group_size, M, K) == 0) return BQ_ERR_UNSUPPORTED;
        if (try_stream_gemv(fmt, group_size, x, one_matrix(wq, sc, bi, y, N), M, K, dev, di, st, workspace,
                            workspace_bytes, &s))
            return s;
        return workspace && workspace_bytes < need ? BQ_ERR_WORKSPACE : BQ_ERR_UNSUPPORTED;
    case BQ_PATH_GEMV:
        if (!has_fast_paths(fmt)) return launch_gemv_affine(fmt, x, wq, sc, bi, y, M, N, K, group_size, st);
        if (stream_gemv_preferred(fmt, M, (N + 15) / 16, K, di.num_sms) &&
            try_stream_gemv(fmt, group_size, x, one_matrix(wq, sc, bi, y, N), M, K, dev, di, st, workspace,
                            workspace_bytes, &s))
            return s;
        if (fmt == WFmt::Q4_0) return launch_gemv<Fmt::Q4_0>(x, wq, sc, bi, y, M, N, K, group_size, st);
        if (fmt == WFmt::AFF4) return launch_gemv<Fmt::AFF4>(x, wq, sc, bi, y, M, N, K, group_size, st);
        return launch_gemv<Fmt::AFF8>(x, wq, sc, bi, y, M, N, K, group_size, st);
    case BQ_PATH_TC_FUSED: {
        // K splits take the caller's workspace when it is large enough, the
        // library's per-device buffer when the caller passed none, and are
        // dropped (one split) when a caller's workspace is too small.
        void* ws = workspace;
        size_t wsb = workspace_bytes;
        if (!ws && need > 0) {
            if ((s = library_workspace(dev, st, need, &ws)) != BQ_OK) return s;
            wsb = need;
        }
        if (fmt == WFmt::Q4_0) return launch_tc<kModeQ4_0>(di, dev, x, wq, sc, bi, y, M, N, K, st, ws, wsb, group_size);
        if (fmt == WFmt::AFF4) return launch_tc<kModeAff4>(di, dev, x, wq, sc, bi, y, M, N, K, st, ws, wsb, group_size);
        return launch_tc<kModeAff8>(di, dev, x, wq, sc, bi, y, M, N, K, st, ws, wsb, group_size);
    }
    default: {
        void* ws = workspace;
        if (!ws && (s = library_workspace(dev, st, need, &ws)) != BQ_OK) return s;
        uint16_t* wb = reinterpret_cast<uint16_t*>(ws);
        s = transpose ? dequant_any(fmt, wq, scales, biases, wb, N, K, group_size, di, st)
                      : dequant_affine_t(fmt, wq, scales, biases, wb, K, N, group_size, di, st);
        if (s != BQ_OK) return s;
        return launch_tc<kModeBF16>(di, dev, x, wb, nullptr, nullptr, y, M, N, K, st);
    }
    }
}

// ------------------------------------------------------------------ allocation-free scratch
// Scratch of quant_matmul_noalloc: the bf16 copy of W that the unfused pair
// stages between its two kernels, as a fixed array of the device image.  Host
// code must not pass the name itself to a kernel (on the host it is a stand-in,
// not a device address); noalloc_scratch looks the address up on the current
// device at every call (no allocation; never stale after a device reset).
static __device__ __align__(256) uint8_t g_noalloc_scratch[BQ_NOALLOC_SCRATCH_BYTES];

bq_status noalloc_scratch(void** out)
{
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
        cudaGetLastError();
        return BQ_ERR_CUDA;
    }
    *out = p;
    return BQ_OK;
}

}  // namespace
}  // namespace bq

using namespace bq;

extern "C" {

bq_status q4_0_dequantize(const uint8_t* wq, const uint16_t* scales_f16, uint16_t* out_bf16, int64_t N, int64_t K,
                          bq_stream_t stream)
{
    if (N < 0 || K < 0 || K % 32 != 0) return BQ_ERR_SHAPE;
    if (N == 0 || K == 0) return BQ_OK;
    if (!wq || !scales_f16 || !out_bf16) return BQ_ERR_NULL;
    if (!aligned16(wq) || !aligned16(scales_f16) || !aligned16(out_bf16)) return BQ_ERR_ALIGN;
    int dev;
    DeviceInfo di;
    bq_status s = current_device(&dev, &di);
    if (s != BQ_OK) return s;
    return dequant_any(WFmt::Q4_0, wq, scales_f16, nullptr, out_bf16, N, K, 32, di, (cudaStream_t)stream);
}

bq_status q4_0_import_aos(const uint8_t* blocks, uint8_t* wq, uint16_t* scales_f16, int64_t N, int64_t K,
                          bq_stream_t stream)
{
    if (N < 0 || K < 0 || K % 32 != 0) return BQ_ERR_SHAPE;
    const int64_t nb = N * (K / 32);
    if (nb == 0) return BQ_OK;
    if (!blocks || !wq || !scales_f16) return BQ_ERR_NULL;
    if (!aligned16(blocks) || !aligned16(wq) || !aligned16(scales_f16)) return BQ_ERR_ALIGN;
    int dev;
    DeviceInfo di;
    bq_status s = current_device(&dev, &di);
    if (s != BQ_OK) return s;
    const int64_t nchunks = (nb + 31) / 32;
    const int64_t grid = std::min<int64_t>((nchunks + kImportWarps - 1) / kImportWarps, (int64_t)di.num_sms * 8);
    q4_0_import_aos_kernel<<<(unsigned)std::max<int64_t>(grid, 1), 32 * kImportWarps, 0, (cudaStream_t)stream>>>(
        blocks, wq, scales_f16, nb);
    return launch_status();
}

bq_status q8_1_quantize(const uint16_t* x_bf16, int8_t* xq, float* dx, int32_t* qsum, int64_t M, int64_t K,
                        bq_stream_t stream)
{
    if (M < 0 || K < 0 || K % 32 != 0) return BQ_ERR_SHAPE;
    const int64_t nb = M * (K / 32);
    if (nb == 0) return BQ_OK;
    if (!x_bf16 || !xq || !dx || !qsum) return BQ_ERR_NULL;
    if (!aligned16(x_bf16) || !aligned16(xq) || !aligned16(dx) || !aligned16(qsum)) return BQ_ERR_ALIGN;
    int dev;
    DeviceInfo di;
    bq_status s = current_device(&dev, &di);
    if (s != BQ_OK) return s;
    q8_1_quantize_kernel<<<grid_for(nb, 128, di), 128, 0, (cudaStream_t)stream>>>(x_bf16, xq, dx, qsum, nb);
    return launch_status();
}

bq_status quant_matmul_q8(const int8_t* xq, const float* dx, const int32_t* qsum, const uint8_t* wq,
                          const uint16_t* scales_f16, uint16_t* y_bf16, int64_t M, int64_t N, int64_t K,
                          bq_stream_t stream)
{
    if (M < 0 || N < 0 || K < 0 || K % 32 != 0) return BQ_ERR_SHAPE;
    if (M == 0 || N == 0) return BQ_OK;
    if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX) return BQ_ERR_SHAPE;
    if (!y_bf16) return BQ_ERR_NULL;
    if (!aligned16(y_bf16)) return BQ_ERR_ALIGN;
    int dev;
    DeviceInfo di;
    bq_status s = current_device(&dev, &di);
    if (s != BQ_OK) return s;
    if (K == 0)
        return cudaMemsetAsync(y_bf16, 0, (size_t)M * (size_t)N * 2u, (cudaStream_t)stream) == cudaSuccess
                   ? BQ_OK : BQ_ERR_CUDA;
    if (!xq || !dx || !qsum || !wq || !scales_f16) return BQ_ERR_NULL;
    if (!aligned16(xq) || !aligned16(dx) || !aligned16(qsum) || !aligned16(wq) || !aligned16(scales_f16))
        return BQ_ERR_ALIGN;
    const int64_t nb = K / 32;
    const unsigned grid = (unsigned)((N + 7) / 8);
    // at most 8 tokens per launch; larger M runs as consecutive token groups
    for (int64_t m0 = 0; m0 < M; m0 += 8) {
        const int mt = (int)std::min<int64_t>(8, M - m0);
        const int8_t* xq_m = xq + m0 * K;
        const float* dx_m = dx + m0 * nb;
        const int32_t* qs_m = qsum + m0 * nb;
        uint16_t* y_m = y_bf16 + m0 * N;
        const cudaStream_t st = (cudaStream_t)stream;
        constexpr int KS = 4;                      // warps per CTA, splitting K
        if (mt == 1)
            gemv_q8_kernel<1, KS><<<grid, 32 * KS, 0, st>>>(xq_m, dx_m, qs_m, wq, scales_f16, y_m, mt, (int)N, (int)K);
        else if (mt == 2)
            gemv_q8_kernel<2, KS><<<grid, 32 * KS, 0, st>>>(xq_m, dx_m, qs_m, wq, scales_f16, y_m, mt, (int)N, (int)K);
        else if (mt <= 4)
            gemv_q8_kernel<4, KS><<<grid, 32 * KS, 0, st>>>(xq_m, dx_m, qs_m, wq, scales_f16, y_m, mt, (int)N, (int)K);
        else
            gemv_q8_kernel<8, KS><<<grid, 32 * KS, 0, st>>>(xq_m, dx_m, qs_m, wq, scales_f16, y_m, mt, (int)N, (int)K);
        if ((s = launch_status()) != BQ_OK) return s;
    }
    return BQ_OK;
}

bq_status affine_dequantize(const uint32_t* wq, const uint16_t* scales_bf16, const uint16_t* biases_bf16,
                            uint16_t* out_bf16, int64_t N, int64_t K, int group_size, int bits, bq_stream_t stream)
{
    WFmt fmt;
    bq_status s = check_format(kAffineTag, N, K, group_size, bits, &fmt);
    if (s != BQ_OK) return s;
    if (N == 0 || K == 0) return BQ_OK;
    if (!wq || !scales_bf16 || !biases_bf16 || !out_bf16) return BQ_ERR_NULL;
    if (!aligned16(wq) || !aligned16(scales_bf16) || !aligned16(biases_bf16) || !aligned16(out_bf16))
        return BQ_ERR_ALIGN;
    int dev;
    DeviceInfo di;
    if ((s = current_device(&dev, &di)) != BQ_OK) return s;
    return dequant_any(fmt, wq, scales_bf16, biases_bf16, out_bf16, N, K, group_size, di, (cudaStream_t)stream);
}

bq_status quant_matmul(const uint16_t* x_bf16, const void* wq, const void* scales, const void* biases,
                       uint16_t* y_bf16, int64_t M, int64_t N, int64_t K, int group_size, int bits, int transpose,
                       bq_stream_t stream)
{
    return matmul_impl(x_bf16, wq, scales, biases, y_bf16, M, N, K, group_size, bits, transpose, BQ_PATH_AUTO,
                       nullptr, 0, (cudaStream_t)stream);
}

bq_status quant_matmul_ex(const uint16_t* x_bf16, const void* wq, const void* scales, const void* biases,
                          uint16_t* y_bf16, int64_t M, int64_t N, int64_t K, int group_size, int bits, int transpose,
                          int path, void* workspace, size_t workspace_bytes, bq_stream_t stream)
{
    return matmul_impl(x_bf16, wq, scales, biases, y_bf16, M, N, K, group_size, bits, transpose, path, workspace,
                       workspace_bytes, (cudaStream_t)stream);
}

bq_status quant_matmul_noalloc(const uint16_t* x_bf16, const void* wq, const void* scales, const void* biases,
                               uint16_t* y_bf16, int64_t M, int64_t N, int64_t K, int group_size, int bits,
                               int transpose, bq_stream_t stream)
{
    if (transpose != 0 && transpose != 1) return BQ_ERR_UNSUPPORTED;
    if (M < 0 || N < 0 || K < 0) return BQ_ERR_SHAPE;
    if (transpose == 0 && !biases) return BQ_ERR_UNSUPPORTED;
    WFmt fmt;
    bq_status s = transpose ? check_format(biases, N, K, group_size, bits, &fmt)
                            : check_format(biases, K, N, group_size, bits, &fmt);
    if (s != BQ_OK) return s;
    if (M == 0 || N == 0 || K == 0)           // nothing to stage: no scratch involved
        return matmul_impl(x_bf16, wq, scales, biases, y_bf16, M, N, K, group_size, bits, transpose,
                           BQ_PATH_DEQUANT_GEMM, nullptr, 0, (cudaStream_t)stream);
    // quant_matmul's own path, with the fixed array as its scratch: the decode
    // GEMV needs none, the fused kernel keeps its K-split partial sums there (or
    // runs unsplit if they do not fit), the unfused pair stages W there.
    const bool gemv_t = transpose == 0 && M <= kGtAutoMaxM && (bits == 2 || bits == 4 || bits == 8);
    const int path = transpose ? select_path(M, K, fmt) : gemv_t ? BQ_PATH_GEMV : BQ_PATH_DEQUANT_GEMM;
    if (path == BQ_PATH_DEQUANT_GEMM && (uint64_t)N > (uint64_t)(BQ_NOALLOC_SCRATCH_BYTES / 2u) / (uint64_t)K)
        return BQ_ERR_WORKSPACE;
    int dev;
    DeviceInfo di;
    if ((s = current_device(&dev, &di)) != BQ_OK) return s;
    void* ws = nullptr;
    if ((s = noalloc_scratch(&ws)) != BQ_OK) return s;
    return matmul_impl(x_bf16, wq, scales, biases, y_bf16, M, N, K, group_size, bits, transpose, path, ws,
                       BQ_NOALLOC_SCRATCH_BYTES, (cudaStream_t)stream);
}

bq_status quant_matmul_multi(const uint16_t* x_bf16, int count, const void* const* wq, const void* const* scales,
                             const void* const* biases, uint16_t* const* y_bf16, const int64_t* N, int64_t M,
                             int64_t K, int group_size, int bits, int transpose, bq_stream_t stream)
{
    if (transpose != 1) return BQ_ERR_UNSUPPORTED;
    if (count < 0 || count > kMultiMax || M < 0 || K < 0) return count > kMultiMax ? BQ_ERR_UNSUPPORTED : BQ_ERR_SHAPE;
    if (count == 0) return BQ_OK;
    if (!wq || !scales || !y_bf16 || !N) return BQ_ERR_NULL;
    WFmt fmt;
    bq_status s;
    for (int i = 0; i < count; ++i) {
        if (N[i] < 0 || N[i] > INT32_MAX) return BQ_ERR_SHAPE;
        if (biases && !biases[i]) return BQ_ERR_NULL;            // all affine or all Q4_0
        if ((s = check_format(biases ? biases[i] : nullptr, N[i], K, group_size, bits, &fmt)) != BQ_OK) return s;
    }
    if (M == 0) return BQ_OK;
    const int path = select_path(M, K, fmt);
    if (path != BQ_PATH_GEMV || K == 0 || !has_fast_paths(fmt)) {
        // prefill sizes: each matrix through its own launch of the chosen path
        for (int i = 0; i < count; ++i) {
            s = matmul_impl(x_bf16, wq[i], scales[i], biases ? biases[i] : nullptr, y_bf16[i], M, N[i], K,
                            group_size, bits, transpose, BQ_PATH_AUTO, nullptr, 0, (cudaStream_t)stream);
            if (s != BQ_OK) return s;
        }
        return BQ_OK;
    }
    if (!x_bf16) return BQ_ERR_NULL;
    if (!aligned16(x_bf16)) return BQ_ERR_ALIGN;
    GemvMultiTable tab;
    tab.count = count;
    for (int i = 0; i < count; ++i) {
        if (N[i] > 0 && (!wq[i] || !scales[i] || !y_bf16[i])) return BQ_ERR_NULL;
        if (N[i] > 0 && (!aligned16(wq[i]) || !aligned16(scales[i]) || !aligned16(y_bf16[i]) ||
                         (biases && !aligned16(biases[i]))))
            return BQ_ERR_ALIGN;
        tab.wq[i] = reinterpret_cast<const uint8_t*>(wq[i]);
        tab.scales[i] = reinterpret_cast<const uint16_t*>(scales[i]);
        tab.biases[i] = biases ? reinterpret_cast<const uint16_t*>(biases[i]) : nullptr;
        tab.y[i] = y_bf16[i];
        tab.N[i] = (int)N[i];
    }
    int dev;
    DeviceInfo di;
    if ((s = current_device(&dev, &di)) != BQ_OK) return s;
    const cudaStream_t st = (cudaStream_t)stream;
    SgMats mats;
    mats.count = count;
    for (int i = 0; i < count; ++i) {
        mats.wq[i] = wq[i];
        mats.scales[i] = tab.scales[i];
        mats.biases[i] = tab.biases[i];
        mats.y[i] = y_bf16[i];
        mats.N[i] = N[i];
    }
    int64_t ntiles_all = 0;
    for (int i = 0; i < count; ++i) ntiles_all += (N[i] + 15) / 16;
    if (stream_gemv_preferred(fmt, M, ntiles_all, K, di.num_sms) &&
        try_stream_gemv(fmt, group_size, x_bf16, mats, M, K, dev, di, st, nullptr, 0, &s))
        return s;
    if (fmt == WFmt::Q4_0) return launch_gemv_multi<Fmt::Q4_0>(x_bf16, tab, M, K, group_size, st);
    if (fmt == WFmt::AFF4) return launch_gemv_multi<Fmt::AFF4>(x_bf16, tab, M, K, group_size, st);
    return launch_gemv_multi<Fmt::AFF8>(x_bf16, tab, M, K, group_size, st);
}

size_t quant_matmul_workspace_size(int64_t M, int64_t N, int64_t K, int group_size, int bits, int path)
{
    WFmt fmt;
    if (M < 0 || check_format(format_tag(group_size, bits), N, K, group_size, bits, &fmt) != BQ_OK) return 0;
    if (path == BQ_PATH_AUTO) path = select_path(M, K, fmt);
    // the current device's SM count and shared memory when there is one, else a B200's
    int dev, num_sms = 148, smem_optin = 232448;
    DeviceInfo di;
    if (cudaGetDevice(&dev) == cudaSuccess && current_device(&dev, &di) == BQ_OK) {
        num_sms = di.num_sms;
        smem_optin = di.max_smem_optin;
    }
    cudaGetLastError();
    return workspace_for(path, fmt, group_size, M, N, K, num_sms, smem_optin);
}

int quant_matmul_gemv_kernel(int64_t M, int64_t N, int64_t K, int group_size, int bits, int path)
{
    WFmt fmt;
    if (M < 1 || check_format(format_tag(group_size, bits), N, K, group_size, bits, &fmt) != BQ_OK) return -1;
    if (path == BQ_PATH_AUTO) path = select_path(M, K, fmt);
    if (path != BQ_PATH_GEMV && path != BQ_PATH_GEMV_STREAM) return -1;
    if (!has_fast_paths(fmt)) return path == BQ_PATH_GEMV && M <= kGaForcedMaxM ? 3 : -1;
    int dev, num_sms = 148, smem_optin = 232448;
    DeviceInfo di;
    if (cudaGetDevice(&dev) == cudaSuccess && current_device(&dev, &di) == BQ_OK) {
        num_sms = di.num_sms;
        smem_optin = di.max_smem_optin;
    }
    cudaGetLastError();
    const bool streamed =
        path == BQ_PATH_GEMV_STREAM || stream_gemv_preferred(fmt, M, (N + 15) / 16, K, num_sms);
    if (streamed && stream_gemv_table_bytes(fmt, group_size, M, K) > 0) {
        SgTmaShape h;
        return tma_shape(fmt, group_size, M, (N + 15) / 16, K, num_sms, smem_optin, &h) ? 1 : 2;
    }
    if (path == BQ_PATH_GEMV_STREAM) return -1;
    return M <= kGemvMaxM ? 0 : -1;
}

int quant_matmul_select_path(int64_t M, int64_t N, int64_t K, int group_size, int bits)
{
    WFmt fmt;
    if (M < 0 || check_format(format_tag(group_size, bits), N, K, group_size, bits, &fmt) != BQ_OK) return -1;
    return select_path(M, K, fmt);
}

bq_status bf16_matmul(const uint16_t* x_bf16, const uint16_t* w_bf16, uint16_t* y_bf16, int64_t M, int64_t N,
                      int64_t K, bq_stream_t stream)
{
    if (M < 0 || N < 0 || K < 0 || K % 8 != 0) return BQ_ERR_SHAPE;
    if (M == 0 || N == 0) return BQ_OK;
    if (!y_bf16) return BQ_ERR_NULL;
    if (!aligned16(y_bf16)) return BQ_ERR_ALIGN;
    int dev;
    DeviceInfo di;
    bq_status s;
    if (K == 0) {
        if ((s = current_device(&dev, &di)) != BQ_OK) return s;
        return cudaMemsetAsync(y_bf16, 0, (size_t)M * N * 2u, (cudaStream_t)stream) == cudaSuccess ? BQ_OK
                                                                                                  : BQ_ERR_CUDA;
    }
    if (!x_bf16 || !w_bf16) return BQ_ERR_NULL;
    if (!aligned16(x_bf16) || !aligned16(w_bf16)) return BQ_ERR_ALIGN;
    if ((s = current_device(&dev, &di)) != BQ_OK) return s;
    return launch_tc<kModeBF16>(di, dev, x_bf16, w_bf16, nullptr, nullptr, y_bf16, M, N, K, (cudaStream_t)stream);
}

bq_status q4_0_quantize(const float* w, uint8_t* wq, uint16_t* scales_f16, int64_t N, int64_t K, bq_stream_t stream)
{
    if (N < 0 || K < 0 || K % 32 != 0) return BQ_ERR_SHAPE;
    const int64_t nb = N * (K / 32);
    if (nb == 0) return BQ_OK;
    if (!w || !wq || !scales_f16) return BQ_ERR_NULL;
    if (!aligned16(w) || !aligned16(wq) || !aligned16(scales_f16)) return BQ_ERR_ALIGN;
    int dev;
    DeviceInfo di;
    bq_status s = current_device(&dev, &di);
    if (s != BQ_OK) return s;
    q4_0_quant_kernel<<<grid_for(nb, 256, di), 256, 0, (cudaStream_t)stream>>>(w, wq, scales_f16, nb);
    return launch_status();
}

bq_status affine_quantize(const float* w, uint32_t* wq, uint16_t* scales_bf16, uint16_t* biases_bf16, int64_t N,
                          int64_t K, int group_size, int bits, bq_stream_t stream)
{
    WFmt fmt;
    bq_status s = check_format(kAffineTag, N, K, group_size, bits, &fmt);
    if (s != BQ_OK) return s;
    const int64_t ng = N * (K / group_size);
    if (ng == 0) return BQ_OK;
    if (!w || !wq || !scales_bf16 || !biases_bf16) return BQ_ERR_NULL;
    if (!aligned16(w) || !aligned16(wq) || !aligned16(scales_bf16) || !aligned16(biases_bf16)) return BQ_ERR_ALIGN;
    int dev;
    DeviceInfo di;
    if ((s = current_device(&dev, &di)) != BQ_OK) return s;
    const int grid = grid_for(ng, 256, di);
    const cudaStream_t st = (cudaStream_t)stream;
    switch (bits) {
    case 2: affine_quant_kernel<2><<<grid, 256, 0, st>>>(w, wq, scales_bf16, biases_bf16, ng, group_size); break;
    case 3: affine_quant_kernel<3><<<grid, 256, 0, st>>>(w, wq, scales_bf16, biases_bf16, ng, group_size); break;
    case 4: affine_quant_kernel<4><<<grid, 256, 0, st>>>(w, wq, scales_bf16, biases_bf16, ng, group_size); break;
    case 6: affine_quant_kernel<6><<<grid, 256, 0, st>>>(w, wq, scales_bf16, biases_bf16, ng, group_size); break;
    default: affine_quant_kernel<8><<<grid, 256, 0, st>>>(w, wq, scales_bf16, biases_bf16, ng, group_size); break;
    }
    return launch_status();
}

// Self-test of the bounded waits: one thread waits on an mbarrier that nothing
// arrives on, with the same try_wait and error recording as the kernels' waits,
// and gives up after limit_cycles SM clocks.
__global__ void selftest_wait_kernel(long long limit_cycles)
{
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x != 0) return;
    const uint32_t b = smem_u32(&bar);
    mbar_init(b, 1);
    fence_barrier_init();
    const long long t0 = clock64();
    while (!mbar_try_wait(b, 0)) {
        if (clock64() - t0 > limit_cycles) {
            raise_device_error(kErrWaitTimeout);
            return;
        }
    }
}

bq_status bq_selftest_wait_timeout(long long limit_cycles, bq_stream_t stream)
{
    if (limit_cycles < 1000 || limit_cycles > 4000000000LL) return BQ_ERR_SHAPE;
    int dev;
    DeviceInfo di;
    bq_status s = current_device(&dev, &di);
    if (s != BQ_OK) return s;
    selftest_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(limit_cycles);
    return launch_status();
}

bq_status bq_device_status(void)
{
    if (cudaDeviceSynchronize() != cudaSuccess) return BQ_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int)) != cudaSuccess) return BQ_ERR_CUDA;
    if (v == 0) return BQ_OK;
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)) != cudaSuccess) return BQ_ERR_CUDA;
    return BQ_ERR_TIMEOUT;
}

const char* bq_status_string(int status)
{
    switch (status) {
    case BQ_OK: return "BQ_OK";
    case BQ_ERR_NULL: return "BQ_ERR_NULL: a required pointer is NULL";
    case BQ_ERR_SHAPE: return "BQ_ERR_SHAPE: invalid size or K not a multiple of the block/group";
    case BQ_ERR_UNSUPPORTED: return "BQ_ERR_UNSUPPORTED: bits/group_size/transpose/path not supported";
    case BQ_ERR_ALIGN: return "BQ_ERR_ALIGN: a device pointer is not 16-byte aligned";
    case BQ_ERR_CUDA: return "BQ_ERR_CUDA: CUDA runtime or launch error";
    case BQ_ERR_TIMEOUT: return "BQ_ERR_TIMEOUT: a device-side bounded wait ran out";
    case BQ_ERR_WORKSPACE: return "BQ_ERR_WORKSPACE: workspace missing or too small";
    case BQ_ERR_DEVICE: return "BQ_ERR_DEVICE: current device is not sm_100";
    default: return "unknown bq_status";
    }
}

int bq_version(void) { return 100; }

}  // extern "C"

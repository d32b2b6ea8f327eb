// cr_lib.cu -- the C ABI of the ConvRot W4A8 codebook linear forward
// (include/cr_w4a8.h): argument validation, per-device state, TMA
// descriptors, and the launches of the sm_100a kernels.
//
// Built as one translation unit (the kernels are header files) into
// libcr_w4a8.so with nvcc -gencode arch=compute_100a,code=sm_100a.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <climits>
#include <functional>
#include <cstdint>
#include <cstring>
#include <new>
#include <mutex>

#include "cr_w4a8.h"
#include "cr_device.cuh"
#include "k_elementwise.cuh"
#include "k_gemm.cuh"
#include "k_gemv.cuh"
#include "k_peak.cuh"
#include "k_quant.cuh"
#include "k_rotquant.cuh"

namespace {

constexpr int kMaxDevices = 64;

struct DeviceState {
    bool probed = false;
    bool usable = false;
    int num_sms = 0;
    cudaMemPool_t pool = nullptr;  // stream-ordered pool for the weight transients (release threshold 0)
    // kernel attributes set once (cudaFuncSetAttribute is idempotent; atomic
    // flags so that concurrent first calls do not race on the flag itself)
    std::atomic<bool> gemm_attr_set{false};
    std::atomic<bool> gemm_pair_attr_set{false};
    std::atomic<bool> gemv_attr_set{false};
    std::atomic<bool> gemv_split_attr_set{false};
    std::atomic<bool> gemv32_attr_set{false};
    std::atomic<bool> gemv32_split_attr_set{false};
    std::atomic<bool> gemv_grouped_attr_set{false};
    std::atomic<bool> gemm_bf16_attr_set{false};
    std::atomic<bool> gemm_pair_bf16_attr_set{false};
    std::atomic<bool> peak_attr_set{false};
    // side stream and events on which cr_w4a8_linear's prefill path decodes
    // the weight while the activations are rotated and quantised
    cudaStream_t side = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
};

DeviceState g_dev[kMaxDevices];
std::mutex g_mutex;

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode_tiled = nullptr;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The driver's tensor-map encoder, looked up once through the runtime (no
// link against libcuda).  Called with g_mutex held.
bool have_encode_tiled()
{
    if (g_encode_tiled != nullptr)
        return true;
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr) {
        cudaGetLastError();
        return false;
    }
    g_encode_tiled = reinterpret_cast<EncodeTiledFn>(fn);
    return true;
}

cr_status check_k(int64_t K)
{
    if (K <= 0 || K % CR_ROT != 0 || K > CR_MAX_K)
        return CR_ERR_UNSUPPORTED;
    return CR_OK;
}

// The current device's state, probing it once.  Fails with CR_ERR_NO_DEVICE
// when there is no usable sm_100 device.
cr_status current_device(DeviceState **out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return CR_ERR_NO_DEVICE;
    }
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceState &d = g_dev[dev];
    if (!d.probed) {
        d.probed = true;
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            cudaGetLastError();
            return CR_ERR_NO_DEVICE;
        }
        d.usable = (major == 10 && minor == 0);
        d.num_sms = sms;
        if (d.usable) {
            cudaMemPoolProps props = {};
            props.allocType = cudaMemAllocationTypePinned;
            props.location.type = cudaMemLocationTypeDevice;
            props.location.id = dev;
            if (cudaMemPoolCreate(&d.pool, &props) != cudaSuccess) {
                cudaGetLastError();
                d.usable = false;
            } else {
                // hold nothing past a synchronisation: a transient's memory
                // goes back to the driver at the next stream, event or device
                // synchronisation after it was freed
                uint64_t keep = 0;
                cudaMemPoolSetAttribute(d.pool, cudaMemPoolAttrReleaseThreshold, &keep);
            }
        }
        if (d.usable && !have_encode_tiled())
            d.usable = false;
        if (d.usable && cr::rq::set_attributes() != cudaSuccess) {
            cudaGetLastError();
            d.usable = false;
        }
    }
    if (!d.usable)
        return CR_ERR_NO_DEVICE;
    *out = &d;
    return CR_OK;
}

cr_status launched(cudaError_t e)
{
    if (e != cudaSuccess)
        return CR_ERR_CUDA;
    return CR_OK;
}

// 2-D int8 tensor map over a row-major [rows, inner] matrix, box
// [box_rows, 128 bytes], 128-byte swizzle; out-of-range rows read as zero.
bool make_tmap_i8(CUtensorMap *map, const void *base, uint64_t inner, uint64_t rows, uint32_t box_rows)
{
    const cuuint64_t dims[2] = {inner, rows};
    const cuuint64_t strides[1] = {inner};
    const cuuint32_t box[2] = {128u, box_rows};
    const cuuint32_t estr[2] = {1u, 1u};
    const CUresult r = g_encode_tiled(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides,
                                      box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 2-D bf16 tensor map for the tcgen05 GEMM: rows of `inner` elements, boxes
// of 64 elements (128 bytes, 128-byte swizzle) x box_rows rows.
bool make_tmap_bf16(CUtensorMap *map, const void *base, uint64_t inner, uint64_t rows, uint32_t box_inner,
                    uint32_t box_rows)
{
    const cuuint64_t dims[2] = {inner, rows};
    const cuuint64_t strides[1] = {inner * 2};
    const cuuint32_t box[2] = {box_inner, box_rows};
    const cuuint32_t estr[2] = {1u, 1u};
    const CUresult r = g_encode_tiled(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims,
                                      strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 3-D tensor map, no swizzle or the 128-byte swizzle, over `base` with the
// given dims (innermost first), the byte strides of dims 1 and 2 and the box.
// The strides need not increase: the maps below reorder a row-major array so
// that a box lands in shared memory in the order the kernel reads it.
bool make_tmap_3d(CUtensorMap *map, const void *base, CUtensorMapDataType dtype, const uint64_t (&dims)[3],
                  const uint64_t (&strides)[2], const uint32_t (&box)[3], bool swizzle128)
{
    const cuuint64_t d[3] = {dims[0], dims[1], dims[2]};
    const cuuint64_t st[2] = {strides[0], strides[1]};
    const cuuint32_t b[3] = {box[0], box[1], box[2]};
    const cuuint32_t estr[3] = {1u, 1u, 1u};
    const CUresult r = g_encode_tiled(map, dtype, 3, const_cast<void *>(base), d, st, b, estr,
                                      CU_TENSOR_MAP_INTERLEAVE_NONE,
                                      swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// The decode GEMV over 1..CR_MAX_LAYERS layers that share the activations
// and the codebook (layers[i].N may be 0).  Layer arguments are already
// checked.  Tensor maps put a stage into shared memory as codes
// [slice][row][64 B] and scales [256-column block][row][16 B] (one pair per
// layer) and activations [slice][token][128 B] (128-byte swizzle); the row
// tiles of all layers are numbered one after the other and run on a
// persistent grid of as many CTAs as fit on the SMs, optionally as a
// programmatic dependent of the previous kernel on the stream.
// The activation map of the decode GEMV over xq [>= M, K], 1 <= M <= 8 (a
// stage's box of M rows x 1024 columns lands as [slice][token][128 B],
// 128-byte swizzle).
bool encode_gemv_x_map(CUtensorMap *map, const int8_t *xq, int64_t M, int64_t K)
{
    if (M < 1 || M > cr::gv::kTokens)
        return false;
    const uint64_t uK = (uint64_t)K;
    return make_tmap_3d(map, xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, {(uint64_t)cr::gv::kSlice, (uint64_t)M,
                                                                   uK / cr::gv::kSlice},
                        {uK, (uint64_t)cr::gv::kSlice},
                        {(uint32_t)cr::gv::kSlice, (uint32_t)M, (uint32_t)(cr::gv::kChunk / cr::gv::kSlice)},
                        true);
}

// Row tile height of a single-layer decode GEMV: 32 rows (two MMA row
// blocks per activation stage) when the layer has at least one such tile per
// SM, 16 otherwise, so that small layers keep more SMs busy.
int gemv_tile_rows(int64_t N, int num_sms)
{
    return (N + 31) / 32 >= num_sms ? 32 : 16;
}

// Everything of a GEMV launch's arguments but the activations (tm_x, xs, M),
// for row tiles of `rows` rows (16, or 32 for a single layer).  `tiles`
// returns the row tiles of all layers (0: nothing to launch).
template <int L>
cr_status build_gemv_args(cr::gv::GemvArgs<L> &args, const float *codebook, int64_t K, const cr_w4a8_layer *layers,
                          int num_layers, cr_out_dtype out_dtype, int swiglu, int64_t &tiles, int rows = 16)
{
    using namespace cr;
    using C = gv::Prod;  // the level-table copies (the same in every configuration)
    static_assert(gv::Prod::kCopies == gv::Prod32::kCopies, "one table stride for both configurations");
    if (rows != 16 && !(rows == 32 && L == 1))
        return CR_ERR_INVALID_ARG;
    memset(&args, 0, sizeof(args));
    const uint64_t uK = (uint64_t)K;
    tiles = 0;
    for (int l = 0; l < num_layers; ++l) {
        const cr_w4a8_layer &ly = layers[l];
        args.layer[l].tile0 = (int)tiles;
        if (ly.N == 0)
            continue; // no tiles; its pointers may be null
        const uint64_t uN = (uint64_t)ly.N;
        if (!make_tmap_3d(&args.tm_codes[l], ly.qdata, CU_TENSOR_MAP_DATA_TYPE_UINT32, {16, uN, uK / gv::kSlice},
                          {uK / 2, 64}, {16, (uint32_t)rows, (uint32_t)(gv::kChunk / gv::kSlice)}, false) ||
            !make_tmap_3d(&args.tm_srel[l], ly.srel, CU_TENSOR_MAP_DATA_TYPE_UINT8, {16, uN, uK / 256}, {uK / 16, 16},
                          {16, (uint32_t)rows, (uint32_t)(gv::kChunk / 256)}, false))
            return CR_ERR_CUDA;
        args.layer[l].ws = ly.s_channel;
        args.layer[l].bias = ly.bias;
        args.layer[l].out = ly.out;
        args.layer[l].acc_out = ly.acc_out;
        args.layer[l].N = (int)ly.N;
        args.layer[l].swiglu = swiglu;
        tiles += (ly.N + rows - 1) / rows;
    }
    if (tiles > INT_MAX)
        return CR_ERR_UNSUPPORTED;
    args.codebook = codebook;
    args.K = (int)K;
    args.num_layers = num_layers;
    args.num_tiles = (int)tiles;
    args.out_f32 = out_dtype == CR_OUT_F32 ? 1 : 0;
    args.lut_step = (uint32_t)(C::kCopies * sizeof(uint4));
    args.ahead = gv::kPrefetchAhead;
    args.tile_rows = rows;
    return CR_OK;
}

// Launch the decode GEMV with complete arguments: a persistent grid of as
// many CTAs as fit on the SMs, optionally as a programmatic dependent of the
// previous kernel on the stream.  split: the layer's tables all have a split
// form (checked when it was prepared); the split variant of the kernel runs
// where every CTA has at most two row tiles.  attr_set / split_attr_set: the
// once-per-device shared-memory attribute of the plain and split variants of
// configuration C.
template <class C, int L>
cr_status launch_gemv_cfg(int num_sms, std::atomic<bool> &attr_set, const cr::gv::GemvArgs<L> &args,
                          cudaStream_t stream, bool pdl, bool split, std::atomic<bool> *split_attr_set)
{
    using namespace cr;
    // persistent grid of several CTAs per SM, at most one wave
    const int64_t slots = (int64_t)C::kMinBlocks * num_sms;
    const int64_t grid = args.num_tiles < slots ? args.num_tiles : slots;
    const bool use_split = split && split_attr_set != nullptr && args.num_tiles <= 2 * grid;
    void (*kern)(const gv::GemvArgs<L>) = use_split ? gv::gemv_kernel<C, L, true> : gv::gemv_kernel<C, L, false>;
    std::atomic<bool> &flag = use_split ? *split_attr_set : attr_set;
    if (!flag) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmemBytes) !=
            cudaSuccess) {
            cudaGetLastError();
            return CR_ERR_CUDA;
        }
        flag = true;
    }
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(gv::kThreads);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return launched(cudaLaunchKernelEx(&cfg, kern, args));
}

// The configuration the arguments were built for (args.tile_rows): 32-row
// tiles need the flags of their own attributes (attr32_set, split32_set).
template <int L>
cr_status launch_gemv_args(int num_sms, std::atomic<bool> &attr_set, const cr::gv::GemvArgs<L> &args,
                           cudaStream_t stream, bool pdl, bool split = false,
                           std::atomic<bool> *split_attr_set = nullptr, std::atomic<bool> *attr32_set = nullptr,
                           std::atomic<bool> *split32_set = nullptr)
{
    if constexpr (L == 1) {
        if (args.tile_rows == 32) {
            if (attr32_set == nullptr)
                return CR_ERR_INVALID_ARG;
            return launch_gemv_cfg<cr::gv::Prod32, 1>(num_sms, *attr32_set, args, stream, pdl, split, split32_set);
        }
    }
    return launch_gemv_cfg<cr::gv::Prod, L>(num_sms, attr_set, args, stream, pdl, split, split_attr_set);
}

// attr32_set: the flag of the 32-row configuration's attribute, or null to
// keep 16-row tiles.
template <int L>
cr_status launch_gemv(int num_sms, std::atomic<bool> &attr_set, const int8_t *xq, const float *xs, const float *codebook,
                      int64_t M, int64_t K, const cr_w4a8_layer *layers, int num_layers, cr_out_dtype out_dtype,
                      cudaStream_t stream, bool pdl, int swiglu = 0, std::atomic<bool> *attr32_set = nullptr)
{
    cr::gv::GemvArgs<L> args;
    int64_t tiles = 0;
    const int rows = (L == 1 && attr32_set != nullptr) ? gemv_tile_rows(layers[0].N, num_sms) : 16;
    cr_status st = build_gemv_args<L>(args, codebook, K, layers, num_layers, out_dtype, swiglu, tiles, rows);
    if (st != CR_OK || tiles == 0)
        return st;
    if (!encode_gemv_x_map(&args.tm_x, xq, M, K))
        return CR_ERR_CUDA;
    args.xs = xs;
    args.M = (int)M;
    return launch_gemv_args<L>(num_sms, attr_set, args, stream, pdl, false, nullptr, attr32_set);
}


cr_status run_gemv_layers(DeviceState &d, const int8_t *xq, const float *xs, const float *codebook, int64_t M,
                          int64_t K, const cr_w4a8_layer *layers, int num_layers, cr_out_dtype out_dtype,
                          cudaStream_t stream, bool pdl)
{
    if (num_layers == 1)
        return launch_gemv<1>(d.num_sms, d.gemv_attr_set, xq, xs, codebook, M, K, layers, 1, out_dtype, stream,
                              pdl, 0, &d.gemv32_attr_set);
    return launch_gemv<cr::gv::kMaxLayers>(d.num_sms, d.gemv_grouped_attr_set, xq, xs, codebook, M, K, layers,
                                           num_layers, out_dtype, stream, pdl);
}

// One layer.
cr_status run_gemv(int num_sms, std::atomic<bool> &attr_set, const int8_t *xq, const float *xs, const uint8_t *qdata,
                   const uint8_t *srel, const float *codebook, const float *s_channel, const float *bias, int64_t M,
                   int64_t N, int64_t K, cr_out_dtype out_dtype, void *out, int32_t *acc_out, cudaStream_t stream,
                   bool pdl, int swiglu = 0, std::atomic<bool> *attr32_set = nullptr)
{
    cr_w4a8_layer ly;
    ly.qdata = qdata;
    ly.srel = srel;
    ly.s_channel = s_channel;
    ly.bias = bias;
    ly.N = N;
    ly.out = out;
    ly.acc_out = acc_out;
    return launch_gemv<1>(num_sms, attr_set, xq, xs, codebook, M, K, &ly, 1, out_dtype, stream, pdl, swiglu,
                          attr32_set);
}

// Shared validation of the contraction entry points.
cr_status check_contraction(const int8_t *xq, const float *xs, const uint8_t *qdata, const uint8_t *srel,
                            const float *codebook, const float *s_channel, const float *bias, int64_t M, int64_t N,
                            int64_t K, cr_out_dtype out_dtype, void *out, int32_t *acc_out)
{
    if (M < 0 || N < 0 || K < 0)
        return CR_ERR_INVALID_ARG;
    if (out_dtype != CR_OUT_BF16 && out_dtype != CR_OUT_F32)
        return CR_ERR_INVALID_ARG;
    const cr_status k = check_k(K);
    if (k != CR_OK)
        return k;
    if (M > INT_MAX || N > INT_MAX)
        return CR_ERR_UNSUPPORTED;
    if (M == 0 || N == 0)
        return CR_OK;
    if (!xq || !xs || !qdata || !srel || !codebook || !s_channel || !out)
        return CR_ERR_INVALID_ARG;
    if (!aligned16(xq) || !aligned16(xs) || !aligned16(qdata) || !aligned16(srel) || !aligned16(codebook) ||
        !aligned16(s_channel) || !aligned16(out) || (bias && !aligned16(bias)) || (acc_out && !aligned16(acc_out)))
        return CR_ERR_ALIGNMENT;
    return CR_OK;
}

// Validation of a layer list: the count, each layer as in check_contraction
// with the shared xq/xs/codebook, and acc_out only where `allow_acc`.
// Output channels of all layers together.
int64_t total_rows(const cr_w4a8_layer *layers, int num_layers)
{
    int64_t n = 0;
    for (int l = 0; l < num_layers; ++l)
        n += layers[l].N;
    return n;
}

static_assert(cr::gv::kMaxLayers == CR_MAX_LAYERS, "layer count of the decode GEMV");

cr_status check_layers(const int8_t *xq, const float *xs, const float *codebook, int64_t M, int64_t K,
                       const cr_w4a8_layer *layers, int num_layers, cr_out_dtype out_dtype, bool allow_acc)
{
    if (!layers || num_layers < 1 || num_layers > CR_MAX_LAYERS)
        return CR_ERR_INVALID_ARG;
    cr_status worst = CR_OK;
    for (int l = 0; l < num_layers; ++l) {
        const cr_w4a8_layer &ly = layers[l];
        if (!allow_acc && ly.acc_out)
            return CR_ERR_INVALID_ARG;
        const cr_status st = check_contraction(xq, xs, ly.qdata, ly.srel, codebook, ly.s_channel, ly.bias, M, ly.N,
                                               K, out_dtype, ly.out, ly.acc_out);
        if (st == CR_ERR_INVALID_ARG || st == CR_ERR_ALIGNMENT)
            return st;
        if (st != CR_OK)
            worst = st;
    }
    return worst;
}

// The side stream and fork/join events of a device, created on first use.
cr_status side_stream(DeviceState &d)
{
    std::lock_guard<std::mutex> lock(g_mutex);
    if (d.side != nullptr)
        return CR_OK;
    cudaStream_t s = nullptr;
    cudaEvent_t f = nullptr, j = nullptr;
    if (cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&f, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&j, cudaEventDisableTiming) != cudaSuccess) {
        cudaGetLastError();
        if (s)
            cudaStreamDestroy(s);
        if (f)
            cudaEventDestroy(f);
        return CR_ERR_CUDA;
    }
    d.side = s;
    d.fork = f;
    d.join = j;
    return CR_OK;
}

// The int8 contraction with the fused epilogue on an int8 weight w8 [N, K]
// (already decoded): tcgen05 GEMM on CTA pairs (256 x 256 tiles) when there
// is at least one tile per SM pair, otherwise one CTA per 128 x 256 tile.
cr_status gemm_on_w8(DeviceState &d, const int8_t *xq, const float *xs, const int8_t *w8, const float *s_channel,
                     const float *bias, int64_t M, int64_t N, int64_t K, cr_out_dtype out_dtype, void *out,
                     int32_t *acc_out, cudaStream_t stream, int swiglu)
{
    using namespace cr;
    cr_status st = CR_OK;
    if (!d.gemm_attr_set) {
        if (cudaFuncSetAttribute(gm::gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)gm::kSmemBytes) != cudaSuccess) {
            cudaGetLastError();
            return CR_ERR_CUDA;
        }
        d.gemm_attr_set = true;
    }
    CUtensorMap ta, tb, to;
    const int out_f32 = out_dtype == CR_OUT_F32;
    const int64_t OC = swiglu ? N / 2 : N;  // output columns
    const int vec_ok = out_f32 ? (OC % 4 == 0) : (OC % 8 == 0);
    // Output through TMA bulk stores when rows are 16-byte multiples and the
    // int32 accumulators are not requested: 32-row x 128-byte boxes, 128B swizzle.
    const int tma_out = vec_ok && acc_out == nullptr;
    if (st == CR_OK && (!make_tmap_i8(&ta, xq, (uint64_t)K, (uint64_t)M, (uint32_t)gm::BM) ||
                        !make_tmap_i8(&tb, w8, (uint64_t)K, (uint64_t)N, (uint32_t)gm::BN)))
        st = CR_ERR_CUDA;
    if (st == CR_OK) {
        to = ta;  // placeholder when the output does not go through TMA
        if (tma_out) {
            const cuuint64_t dims[2] = {(cuuint64_t)OC, (cuuint64_t)M};
            const cuuint64_t strides[1] = {(cuuint64_t)OC * (out_f32 ? 4u : 2u)};
            const cuuint32_t box[2] = {out_f32 ? 32u : 64u, 32u};
            const cuuint32_t estr[2] = {1u, 1u};
            if (g_encode_tiled(&to, out_f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, out,
                               dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
                st = CR_ERR_CUDA;
        }
    }
    const int64_t pair_tiles = ((M + 255) / 256) * ((N + gm::BN - 1) / gm::BN);
    const bool use_pair = pair_tiles >= d.num_sms / 2;
    if (st == CR_OK && use_pair) {
        CUtensorMap tb_half;
        if (!d.gemm_pair_attr_set) {
            if (cudaFuncSetAttribute(gm::gemm_pair_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)gm::pair::kSmemBytes) != cudaSuccess) {
                cudaGetLastError();
                st = CR_ERR_CUDA;
            } else {
                d.gemm_pair_attr_set = true;
            }
        }
        if (st == CR_OK && !make_tmap_i8(&tb_half, w8, (uint64_t)K, (uint64_t)N, 128u))
            st = CR_ERR_CUDA;
        if (st == CR_OK) {
            const int64_t pairs = pair_tiles < d.num_sms / 2 ? pair_tiles : d.num_sms / 2;
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3((unsigned)(2 * pairs));
            cfg.blockDim = dim3(gm::kThreads);
            cfg.dynamicSmemBytes = gm::pair::kSmemBytes;
            cfg.stream = stream;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = 2;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            st = launched(cudaLaunchKernelEx(&cfg, gm::gemm_pair_kernel<false>, ta, tb_half, to, xs, s_channel, bias, (int)M,
                                             (int)N, (int)K, out_f32, swiglu, tma_out, out, acc_out));
        }
    } else if (st == CR_OK) {
        const int64_t tiles = ((M + gm::BM - 1) / gm::BM) * ((N + gm::BN - 1) / gm::BN);
        const int grid = (int)(tiles < d.num_sms ? tiles : d.num_sms);
        gm::gemm_kernel<false><<<grid, gm::kThreads, gm::kSmemBytes, stream>>>(ta, tb, to, xs, s_channel, bias, (int)M,
                                                                         (int)N, (int)K, out_f32, swiglu, tma_out, out,
                                                                         acc_out);
        st = launched(cudaGetLastError());
    }
    return st;
}

// The prefill contraction.  When `activations` is given (cr_w4a8_linear), it
// launches the activation kernel on `stream` while the weight decode runs on
// the device's side stream (the two are independent); the GEMM waits for both.
// The weight is decoded into the caller's w8_work [N, K] when given, otherwise
// into a transient from the device's stream-ordered pool, freed on `stream`
// after the GEMM.
cr_status run_gemm(DeviceState &d, const int8_t *xq, const float *xs, const uint8_t *qdata, const uint8_t *srel,
                   const float *codebook, const float *s_channel, const float *bias, int64_t M, int64_t N, int64_t K,
                   cr_out_dtype out_dtype, void *out, int32_t *acc_out, cudaStream_t stream,
                   const std::function<cr_status()> *activations = nullptr, int swiglu = 0,
                   int8_t *w8_work = nullptr)
{
    using namespace cr;
    // The int8 grid of the weight, decoded once per call.
    int8_t *w8 = w8_work;
    if (w8 == nullptr &&
        cudaMallocFromPoolAsync(reinterpret_cast<void **>(&w8), (size_t)(N * K), d.pool, stream) != cudaSuccess) {
        cudaGetLastError();
        return CR_ERR_CUDA;
    }
    cr_status st = CR_OK;
    if (activations != nullptr) {
        st = side_stream(d);
        if (st == CR_OK && (cudaEventRecord(d.fork, stream) != cudaSuccess ||
                            cudaStreamWaitEvent(d.side, d.fork, 0) != cudaSuccess)) {
            cudaGetLastError();
            st = CR_ERR_CUDA;
        }
        if (st == CR_OK)
            st = launched(ew::launch_decode(qdata, srel, codebook, N, K, w8, d.num_sms, d.side));
        if (st == CR_OK && cudaEventRecord(d.join, d.side) != cudaSuccess) {
            cudaGetLastError();
            st = CR_ERR_CUDA;
        }
        if (st == CR_OK)
            st = (*activations)();
        if (st == CR_OK && cudaStreamWaitEvent(stream, d.join, 0) != cudaSuccess) {
            cudaGetLastError();
            st = CR_ERR_CUDA;
        }
    } else {
        st = launched(ew::launch_decode(qdata, srel, codebook, N, K, w8, d.num_sms, stream));
    }
    if (st == CR_OK)
        st = gemm_on_w8(d, xq, xs, w8, s_channel, bias, M, N, K, out_dtype, out, acc_out, stream, swiglu);
    if (w8_work == nullptr && cudaFreeAsync(w8, stream) != cudaSuccess) {
        cudaGetLastError();
        if (st == CR_OK)
            st = CR_ERR_CUDA;
    }
    return st;
}

}  // namespace

// The result word of split_check_kernel (one per device; checks are
// serialised under g_mutex).
static __device__ int g_split_bad = 0;

namespace {
// Whether every scale byte of a layer srel [N, K / 16] has a split table for
// this codebook: split_check_kernel on the legacy default stream, waited for.
cr_status check_split(DeviceState &d, const uint8_t *srel, const float *codebook, int64_t N, int64_t K, bool &ok)
{
    ok = false;
    std::lock_guard<std::mutex> lock(g_mutex);
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_split_bad, &zero, sizeof(int)) != cudaSuccess) {
        cudaGetLastError();
        return CR_ERR_CUDA;
    }
    void *flag = nullptr;
    if (cudaGetSymbolAddress(&flag, g_split_bad) != cudaSuccess) {
        cudaGetLastError();
        return CR_ERR_CUDA;
    }
    const int64_t bytes = N * (K / 16);
    const int64_t words = bytes / 16;
    int64_t grid = (words + 255) / 256;
    if (grid > 2 * (int64_t)d.num_sms)
        grid = 2 * (int64_t)d.num_sms;
    if (grid < 1)
        grid = 1;
    cr::gv::split_check_kernel<<<(unsigned)grid, 256>>>(srel, bytes, codebook, static_cast<int *>(flag));
    int bad = 1;
    if (cudaGetLastError() != cudaSuccess || cudaMemcpyFromSymbol(&bad, g_split_bad, sizeof(int)) != cudaSuccess) {
        cudaGetLastError();
        return CR_ERR_CUDA;
    }
    ok = bad == 0;
    return CR_OK;
}
}  // namespace

// A prepared layer (cr_w4a8_plan_*): the validated layer, its device, and
// the decode GEMV's arguments with the weight maps encoded; tm_x holds the
// activation map of (xmap_base, xmap_M) once a forward has set it.
struct cr_w4a8_plan_st {
    int device = -1;
    DeviceState *d = nullptr;
    const uint8_t *qdata = nullptr, *srel = nullptr;
    const float *codebook = nullptr, *s_channel = nullptr, *bias = nullptr;
    int64_t N = 0, K = 0;
    int act_qmax = 127;
    cr_out_dtype out_dtype = CR_OUT_BF16;
    cr::gv::GemvArgs<1> gemv;
    int64_t tiles = 0;
    bool split_ok = false;  // every scale byte of the layer has a split table (split_check_kernel)
    const int8_t *xmap_base = nullptr;
    int64_t xmap_M = -1;
    std::mutex mu;
};

// A host-buffer forward bound to its buffers (cr_w4a8_plan_bind_host): the
// checks, the host mappings and the decode GEMV's complete arguments are
// resolved once; a run only queues the launches.
struct cr_w4a8_host_call_st {
    cr_w4a8_plan plan = nullptr;
    const uint16_t *x_host = nullptr;
    void *out_host = nullptr;
    const void *x_map = nullptr;  // device address of x_host (copied by a kernel), or null (copy engine)
    void *out_map = nullptr;      // the same for out_host (a decode batch's GEMV stores into it directly)
    uint16_t *x_dev = nullptr;
    void *out_dev = nullptr;
    int8_t *xq = nullptr;
    float *xs = nullptr;
    int64_t M = 0, MP = 0;
    size_t xb = 0, ob = 0;
    cr::gv::GemvArgs<1> gemv;  // M <= CR_GEMV_MAX_M: the GEMV launch's arguments, activation map included
};

extern "C" {

const char *cr_status_string(cr_status s)
{
    switch (s) {
    case CR_OK: return "ok";
    case CR_ERR_INVALID_ARG: return "invalid argument";
    case CR_ERR_UNSUPPORTED: return "unsupported shape";
    case CR_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case CR_ERR_CUDA: return "CUDA runtime or launch failure";
    case CR_ERR_TIMEOUT: return "device pipeline wait timed out";
    case CR_ERR_NO_DEVICE: return "no usable sm_100 device";
    }
    return "unknown status";
}

const char *cr_version(void) { return "0.1.0"; }

cr_status cr_rotate_quant_act(const uint16_t *x, int64_t M, int64_t K, int64_t MP, int act_qmax, int8_t *xq, float *xs,
                              cr_stream_t stream)
{
    if (M < 0 || K < 0 || MP < M || act_qmax < 1 || act_qmax > 127)
        return CR_ERR_INVALID_ARG;
    const cr_status k = check_k(K);
    if (k != CR_OK)
        return k;
    if (MP > INT_MAX)
        return CR_ERR_UNSUPPORTED;
    if (MP == 0)
        return CR_OK;
    if ((M > 0 && !x) || !xq || !xs)
        return CR_ERR_INVALID_ARG;
    if ((x && !aligned16(x)) || !aligned16(xq) || !aligned16(xs))
        return CR_ERR_ALIGNMENT;
    DeviceState *d = nullptr;
    const cr_status ds = current_device(&d);
    if (ds != CR_OK)
        return ds;
    return launched(cr::rq::launch(x, M, K, MP, act_qmax, xq, xs, stream));
}

cr_status cr_w4a8_decode_int8(const uint8_t *qdata, const uint8_t *srel, const float *codebook, int64_t N, int64_t K,
                              int8_t *w8, cr_stream_t stream)
{
    if (N < 0 || K < 0)
        return CR_ERR_INVALID_ARG;
    const cr_status k = check_k(K);
    if (k != CR_OK)
        return k;
    if (N == 0)
        return CR_OK;
    if (!qdata || !srel || !codebook || !w8)
        return CR_ERR_INVALID_ARG;
    if (!aligned16(qdata) || !aligned16(srel) || !aligned16(codebook) || !aligned16(w8))
        return CR_ERR_ALIGNMENT;
    DeviceState *d = nullptr;
    const cr_status ds = current_device(&d);
    if (ds != CR_OK)
        return ds;
    return launched(cr::ew::launch_decode(qdata, srel, codebook, N, K, w8, d->num_sms, stream));
}

cr_status cr_w4a8_gemm(const int8_t *xq, const float *xs, const uint8_t *qdata, const uint8_t *srel,
                       const float *codebook, const float *s_channel, const float *bias, int64_t M, int64_t N,
                       int64_t K, cr_out_dtype out_dtype, void *out, int32_t *acc_out, cr_stream_t stream)
{
    cr_status st = check_contraction(xq, xs, qdata, srel, codebook, s_channel, bias, M, N, K, out_dtype, out, acc_out);
    if (st != CR_OK || M == 0 || N == 0)
        return st;
    DeviceState *d = nullptr;
    st = current_device(&d);
    if (st != CR_OK)
        return st;
    return run_gemm(*d, xq, xs, qdata, srel, codebook, s_channel, bias, M, N, K, out_dtype, out, acc_out, stream);
}

cr_status cr_w4a8_gemm_ws(const int8_t *xq, const float *xs, const uint8_t *qdata, const uint8_t *srel,
                          const float *codebook, const float *s_channel, const float *bias, int64_t M, int64_t N,
                          int64_t K, cr_out_dtype out_dtype, void *out, int32_t *acc_out, int8_t *w8_work,
                          cr_stream_t stream)
{
    cr_status st = check_contraction(xq, xs, qdata, srel, codebook, s_channel, bias, M, N, K, out_dtype, out, acc_out);
    if (st != CR_OK || M == 0 || N == 0)
        return st;
    if (!w8_work)
        return CR_ERR_INVALID_ARG;
    if (!aligned16(w8_work))
        return CR_ERR_ALIGNMENT;
    DeviceState *d = nullptr;
    st = current_device(&d);
    if (st != CR_OK)
        return st;
    return run_gemm(*d, xq, xs, qdata, srel, codebook, s_channel, bias, M, N, K, out_dtype, out, acc_out, stream,
                    nullptr, 0, w8_work);
}

cr_status cr_w4a8_gemv(const int8_t *xq, const float *xs, const uint8_t *qdata, const uint8_t *srel,
                       const float *codebook, const float *s_channel, const float *bias, int64_t M, int64_t N,
                       int64_t K, cr_out_dtype out_dtype, void *out, int32_t *acc_out, cr_stream_t stream)
{
    if (M > CR_GEMV_MAX_M)
        return CR_ERR_UNSUPPORTED;
    cr_status st = check_contraction(xq, xs, qdata, srel, codebook, s_channel, bias, M, N, K, out_dtype, out, acc_out);
    if (st != CR_OK || M == 0 || N == 0)
        return st;
    DeviceState *d = nullptr;
    st = current_device(&d);
    if (st != CR_OK)
        return st;
    return run_gemv(d->num_sms, d->gemv_attr_set, xq, xs, qdata, srel, codebook, s_channel, bias, M, N, K,
                    out_dtype, out, acc_out, stream, /*pdl=*/true, 0, &d->gemv32_attr_set);
}

cr_status cr_epilogue(const int32_t *acc, const float *xs, const float *s_channel, const float *bias, int64_t M,
                      int64_t N, cr_out_dtype out_dtype, void *out, cr_stream_t stream)
{
    if (M < 0 || N < 0 || (out_dtype != CR_OUT_BF16 && out_dtype != CR_OUT_F32))
        return CR_ERR_INVALID_ARG;
    if (M == 0 || N == 0)
        return CR_OK;
    if (!acc || !xs || !s_channel || !out)
        return CR_ERR_INVALID_ARG;
    if (!aligned16(acc) || !aligned16(xs) || !aligned16(s_channel) || !aligned16(out) || (bias && !aligned16(bias)))
        return CR_ERR_ALIGNMENT;
    DeviceState *d = nullptr;
    const cr_status ds = current_device(&d);
    if (ds != CR_OK)
        return ds;
    return launched(cr::ew::launch_epilogue(acc, xs, s_channel, bias, M, N, out_dtype == CR_OUT_F32, out, d->num_sms,
                                            stream));
}

}  // extern "C"

namespace {

// cr_w4a8_linear and cr_w4a8_linear_swiglu: rotate + quantise, then the GEMV
// (M <= 8) or the GEMM with the weight decode overlapping the activations.
// With ws_given, the prefill path (M > 8) decodes the weight into the
// caller's w8_work [N, K] (which must then be given) instead of a pool
// transient.
cr_status linear_impl(const uint16_t *x, const uint8_t *qdata, const uint8_t *srel, const float *codebook,
                      const float *s_channel, const float *bias, int64_t M, int64_t N, int64_t K, int act_qmax,
                      cr_out_dtype out_dtype, void *out, int8_t *xq_work, float *xs_work, cudaStream_t stream,
                      int swiglu, bool ws_given = false, int8_t *w8_work = nullptr)
{
    if (M < 0 || N < 0 || K < 0 || act_qmax < 1 || act_qmax > 127)
        return CR_ERR_INVALID_ARG;
    if (swiglu && N % 2 != 0)
        return CR_ERR_INVALID_ARG;
    int64_t MP = M;
    if (M >= 1 && M <= CR_GEMV_MAX_M) {
        MP = 1;
        while (MP < M)
            MP <<= 1;
    }
    cr_status st = check_contraction(xq_work, xs_work, qdata, srel, codebook, s_channel, bias, M, N, K, out_dtype,
                                      out, nullptr);
    if (st != CR_OK || M == 0 || N == 0)
        return st;
    if (!x)
        return CR_ERR_INVALID_ARG;
    if (!aligned16(x))
        return CR_ERR_ALIGNMENT;
    if (ws_given && M > CR_GEMV_MAX_M) {
        if (!w8_work)
            return CR_ERR_INVALID_ARG;
        if (!aligned16(w8_work))
            return CR_ERR_ALIGNMENT;
    }
    DeviceState *d = nullptr;
    st = current_device(&d);
    if (st != CR_OK)
        return st;
    auto activations = [&]() { return launched(cr::rq::launch(x, M, K, MP, act_qmax, xq_work, xs_work, stream)); };
    if (M > CR_GEMV_MAX_M) {
        const std::function<cr_status()> act = activations;
        return run_gemm(*d, xq_work, xs_work, qdata, srel, codebook, s_channel, bias, M, N, K, out_dtype, out, nullptr,
                        stream, &act, swiglu, ws_given ? w8_work : nullptr);
    }
    st = activations();
    if (st != CR_OK)
        return st;
    return run_gemv(d->num_sms, d->gemv_attr_set, xq_work, xs_work, qdata, srel, codebook, s_channel, bias, M, N, K,
                    out_dtype, out, nullptr, stream, /*pdl=*/true, swiglu, &d->gemv32_attr_set);
}

// cr_w4a8_gemm_swiglu and cr_w4a8_gemv_swiglu.
cr_status contraction_swiglu(bool gemv, const int8_t *xq, const float *xs, const uint8_t *qdata, const uint8_t *srel,
                             const float *codebook, const float *s_channel, const float *bias, int64_t M, int64_t N,
                             int64_t K, cr_out_dtype out_dtype, void *out, cudaStream_t stream)
{
    if (gemv && M > CR_GEMV_MAX_M)
        return CR_ERR_UNSUPPORTED;
    if (N % 2 != 0)
        return CR_ERR_INVALID_ARG;
    cr_status st = check_contraction(xq, xs, qdata, srel, codebook, s_channel, bias, M, N, K, out_dtype, out, nullptr);
    if (st != CR_OK || M == 0 || N == 0)
        return st;
    DeviceState *d = nullptr;
    st = current_device(&d);
    if (st != CR_OK)
        return st;
    if (gemv)
        return run_gemv(d->num_sms, d->gemv_attr_set, xq, xs, qdata, srel, codebook, s_channel, bias, M, N, K,
                        out_dtype, out, nullptr, stream, /*pdl=*/true, /*swiglu=*/1, &d->gemv32_attr_set);
    return run_gemm(*d, xq, xs, qdata, srel, codebook, s_channel, bias, M, N, K, out_dtype, out, nullptr, stream,
                    nullptr, /*swiglu=*/1);
}

// The device address of host buffer [p, p + bytes) when it is at most
// kHostCopyMax bytes, 16-byte aligned, a multiple of 16 bytes long, and both
// its first and last byte lie in page-locked host memory mapped for the
// device at addresses `bytes - 1` apart; otherwise null.
constexpr size_t kHostCopyMax = 1u << 20;

// Whether a host-buffer forward's decode GEMV stores y into the mapped
// out_host itself: a decode batch with bf16 outputs whose every full row tile
// leaves as 16-byte stores (N a multiple of 8).  Other outputs would cross the
// host link as scattered 2- or 4-byte stores, and the copy kernel moves them.
bool gemv_stores_host(const cr_w4a8_plan_st *plan, int64_t M)
{
    return M <= CR_GEMV_MAX_M && plan->out_dtype == CR_OUT_BF16 && plan->N % 8 == 0;
}

const void *small_mapped_host(const void *p, size_t bytes)
{
    if (bytes == 0 || bytes > kHostCopyMax || bytes % 16 != 0 || !aligned16(p))
        return nullptr;
    cudaPointerAttributes a0, a1;
    const char *last = static_cast<const char *>(p) + bytes - 1;
    if (cudaPointerGetAttributes(&a0, p) != cudaSuccess || cudaPointerGetAttributes(&a1, last) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    if (a0.type != cudaMemoryTypeHost || a1.type != cudaMemoryTypeHost || !a0.devicePointer || !a1.devicePointer)
        return nullptr;
    if (static_cast<const char *>(a1.devicePointer) - static_cast<const char *>(a0.devicePointer) !=
        (ptrdiff_t)(bytes - 1))
        return nullptr;
    return a0.devicePointer;
}

}  // namespace

extern "C" {

cr_status cr_w4a8_linear(const uint16_t *x, const uint8_t *qdata, const uint8_t *srel, const float *codebook,
                         const float *s_channel, const float *bias, int64_t M, int64_t N, int64_t K, int act_qmax,
                         cr_out_dtype out_dtype, void *out, int8_t *xq_work, float *xs_work, cr_stream_t stream)
{
    return linear_impl(x, qdata, srel, codebook, s_channel, bias, M, N, K, act_qmax, out_dtype, out, xq_work, xs_work,
                       stream, 0);
}

cr_status cr_w4a8_linear_ws(const uint16_t *x, const uint8_t *qdata, const uint8_t *srel, const float *codebook,
                            const float *s_channel, const float *bias, int64_t M, int64_t N, int64_t K, int act_qmax,
                            cr_out_dtype out_dtype, void *out, int8_t *xq_work, float *xs_work, int8_t *w8_work,
                            cr_stream_t stream)
{
    return linear_impl(x, qdata, srel, codebook, s_channel, bias, M, N, K, act_qmax, out_dtype, out, xq_work, xs_work,
                       stream, 0, /*ws_given=*/true, w8_work);
}

cr_status cr_w4a8_linear_swiglu(const uint16_t *x, const uint8_t *qdata, const uint8_t *srel, const float *codebook,
                                const float *s_channel, const float *bias, int64_t M, int64_t N, int64_t K,
                                int act_qmax, cr_out_dtype out_dtype, void *out, int8_t *xq_work, float *xs_work,
                                cr_stream_t stream)
{
    return linear_impl(x, qdata, srel, codebook, s_channel, bias, M, N, K, act_qmax, out_dtype, out, xq_work, xs_work,
                       stream, 1);
}

cr_status cr_w4a8_gemm_swiglu(const int8_t *xq, const float *xs, const uint8_t *qdata, const uint8_t *srel,
                              const float *codebook, const float *s_channel, const float *bias, int64_t M, int64_t N,
                              int64_t K, cr_out_dtype out_dtype, void *out, cr_stream_t stream)
{
    return contraction_swiglu(false, xq, xs, qdata, srel, codebook, s_channel, bias, M, N, K, out_dtype, out, stream);
}

cr_status cr_w4a8_gemv_swiglu(const int8_t *xq, const float *xs, const uint8_t *qdata, const uint8_t *srel,
                              const float *codebook, const float *s_channel, const float *bias, int64_t M, int64_t N,
                              int64_t K, cr_out_dtype out_dtype, void *out, cr_stream_t stream)
{
    return contraction_swiglu(true, xq, xs, qdata, srel, codebook, s_channel, bias, M, N, K, out_dtype, out, stream);
}

namespace {
// Validation shared by the backward entry points: K as for the forward, N a
// multiple of 8 (16-byte rows of the bf16 operands), 16-byte aligned buffers.
cr_status check_backward(const uint8_t *qdata, const uint8_t *srel, const float *codebook, const float *s_channel,
                         int64_t N, int64_t K, const void *a, const void *b, bool empty = false)
{
    if (N < 0 || K < 0)
        return CR_ERR_INVALID_ARG;
    const cr_status k = check_k(K);
    if (k != CR_OK)
        return k;
    if (N % 8 != 0 || N > INT_MAX)
        return CR_ERR_UNSUPPORTED;
    if (N == 0 || empty)
        return CR_OK;
    if (!qdata || !srel || !codebook || !s_channel || !a || !b)
        return CR_ERR_INVALID_ARG;
    if (!aligned16(qdata) || !aligned16(srel) || !aligned16(codebook) || !aligned16(s_channel) || !aligned16(a) ||
        !aligned16(b))
        return CR_ERR_ALIGNMENT;
    return CR_OK;
}
}  // namespace

cr_status cr_w4a8_dequant_t_bf16(const uint8_t *qdata, const uint8_t *srel, const float *codebook,
                                 const float *s_channel, int64_t N, int64_t K, uint16_t *wt, cr_stream_t stream)
{
    cr_status st = check_backward(qdata, srel, codebook, s_channel, N, K, wt, wt);
    if (st != CR_OK || N == 0)
        return st;
    DeviceState *d = nullptr;
    st = current_device(&d);
    if (st != CR_OK)
        return st;
    return launched(cr::ew::launch_dequant_t_bf16(qdata, srel, codebook, s_channel, (int)N, (int)K, wt, d->num_sms,
                                                  stream));
}

namespace {
// cr_w4a8_ste_backward(_ws): wt_work [K, N] bf16 is the caller's transient
// when ws_given (it must then be given), otherwise one from the pool.
cr_status ste_backward_impl(const uint16_t *grad, const uint8_t *qdata, const uint8_t *srel,
                            const float *codebook, const float *s_channel, int64_t M, int64_t N, int64_t K,
                            uint16_t *dx, cudaStream_t stream, bool ws_given, uint16_t *wt_work)
{
    if (M < 0)
        return CR_ERR_INVALID_ARG;
    if (M > INT_MAX)
        return CR_ERR_UNSUPPORTED;
    cr_status st = check_backward(qdata, srel, codebook, s_channel, N, K, grad, dx, /*empty=*/M == 0);
    if (st != CR_OK || M == 0)
        return st;
    if (N == 0) {  // an empty sum: dx = 0
        if (!dx)
            return CR_ERR_INVALID_ARG;
        return cudaMemsetAsync(dx, 0, (size_t)(M * K) * 2, stream) == cudaSuccess ? CR_OK : CR_ERR_CUDA;
    }
    if (ws_given) {
        if (!wt_work)
            return CR_ERR_INVALID_ARG;
        if (!aligned16(wt_work))
            return CR_ERR_ALIGNMENT;
    }
    DeviceState *d = nullptr;
    st = current_device(&d);
    if (st != CR_OK)
        return st;
    using namespace cr;
    if (!d->gemm_bf16_attr_set) {
        if (cudaFuncSetAttribute(gm::gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)gm::kSmemBytes) != cudaSuccess) {
            cudaGetLastError();
            return CR_ERR_CUDA;
        }
        d->gemm_bf16_attr_set = true;
    }
    // the transposed bf16 weight: the caller's transient, or one from the
    // stream-ordered pool
    uint16_t *wt = wt_work;
    if (!ws_given &&
        cudaMallocFromPoolAsync(reinterpret_cast<void **>(&wt), (size_t)(N * K) * 2, d->pool, stream) != cudaSuccess) {
        cudaGetLastError();
        return CR_ERR_CUDA;
    }
    st = launched(ew::launch_dequant_t_bf16(qdata, srel, codebook, s_channel, (int)N, (int)K, wt, d->num_sms, stream));
    // dx [M, K] = grad [M, N] x wt [K, N]^T: the GEMM's rows are M, its columns K, its reduction N
    CUtensorMap ta, tb, to;
    if (st == CR_OK && (!make_tmap_bf16(&ta, grad, (uint64_t)N, (uint64_t)M, 64u, (uint32_t)gm::BM) ||
                        !make_tmap_bf16(&tb, wt, (uint64_t)N, (uint64_t)K, 64u, (uint32_t)gm::BN) ||
                        !make_tmap_bf16(&to, dx, (uint64_t)K, (uint64_t)M, 64u, 32u)))
        st = CR_ERR_CUDA;
    // 256 x 256 tiles on CTA pairs when there is at least one per SM pair
    const int64_t pair_tiles = ((M + 255) / 256) * ((K + gm::BN - 1) / gm::BN);
    if (st == CR_OK && pair_tiles >= d->num_sms / 2) {
        CUtensorMap tb_half;
        if (!d->gemm_pair_bf16_attr_set) {
            if (cudaFuncSetAttribute(gm::gemm_pair_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)gm::pair::kSmemBytes) != cudaSuccess) {
                cudaGetLastError();
                st = CR_ERR_CUDA;
            } else {
                d->gemm_pair_bf16_attr_set = true;
            }
        }
        if (st == CR_OK && !make_tmap_bf16(&tb_half, wt, (uint64_t)N, (uint64_t)K, 64u, 128u))
            st = CR_ERR_CUDA;
        if (st == CR_OK) {
            const int64_t pairs = pair_tiles < d->num_sms / 2 ? pair_tiles : d->num_sms / 2;
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3((unsigned)(2 * pairs));
            cfg.blockDim = dim3(gm::kThreads);
            cfg.dynamicSmemBytes = gm::pair::kSmemBytes;
            cfg.stream = stream;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = 2;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            st = launched(cudaLaunchKernelEx(&cfg, gm::gemm_pair_kernel<true>, ta, tb_half, to, (const float *)nullptr,
                                             (const float *)nullptr, (const float *)nullptr, (int)M, (int)K, (int)N,
                                             0, 0, 1, (void *)dx, (int32_t *)nullptr));
        }
    } else if (st == CR_OK) {
        const int64_t tiles = ((M + gm::BM - 1) / gm::BM) * ((K + gm::BN - 1) / gm::BN);
        const int grid = (int)(tiles < d->num_sms ? tiles : d->num_sms);
        gm::gemm_kernel<true><<<grid, gm::kThreads, gm::kSmemBytes, stream>>>(
            ta, tb, to, nullptr, nullptr, nullptr, (int)M, (int)K, (int)N, /*out_f32=*/0, /*swiglu=*/0,
            /*tma_out=*/1, dx, nullptr);
        st = launched(cudaGetLastError());
    }
    if (!ws_given && cudaFreeAsync(wt, stream) != cudaSuccess) {
        cudaGetLastError();
        if (st == CR_OK)
            st = CR_ERR_CUDA;
    }
    return st;
}
}  // namespace

cr_status cr_w4a8_ste_backward(const uint16_t *grad, const uint8_t *qdata, const uint8_t *srel,
                               const float *codebook, const float *s_channel, int64_t M, int64_t N, int64_t K,
                               uint16_t *dx, cr_stream_t stream)
{
    return ste_backward_impl(grad, qdata, srel, codebook, s_channel, M, N, K, dx, stream, false, nullptr);
}

cr_status cr_w4a8_ste_backward_ws(const uint16_t *grad, const uint8_t *qdata, const uint8_t *srel,
                                  const float *codebook, const float *s_channel, int64_t M, int64_t N, int64_t K,
                                  uint16_t *dx, uint16_t *wt_work, cr_stream_t stream)
{
    return ste_backward_impl(grad, qdata, srel, codebook, s_channel, M, N, K, dx, stream, true, wt_work);
}

namespace {
// Validation shared by the quantiser entry points: N >= 0, K a positive
// multiple of 16 up to CR_MAX_K, 16-byte aligned non-null buffers.
cr_status check_quant(const float *w_rot, const float *codebook, int64_t N, int64_t K, const void *a, const void *b,
                      const void *c)
{
    if (N < 0 || K < 0)
        return CR_ERR_INVALID_ARG;
    if (K == 0 || K % 16 != 0 || K > CR_MAX_K)
        return CR_ERR_UNSUPPORTED;
    if (N == 0)
        return CR_OK;
    if (!w_rot || !codebook || !a || !b || !c)
        return CR_ERR_INVALID_ARG;
    if (!aligned16(w_rot) || !aligned16(codebook) || !aligned16(a) || !aligned16(b) || !aligned16(c))
        return CR_ERR_ALIGNMENT;
    return CR_OK;
}
}  // namespace

cr_status cr_w4a8_quantize_rotated(const float *w_rot, const float *codebook, int64_t N, int64_t K, uint8_t *qdata,
                                   uint8_t *srel, float *s_channel, cr_stream_t stream)
{
    cr_status st = check_quant(w_rot, codebook, N, K, qdata, srel, s_channel);
    if (st != CR_OK || N == 0)
        return st;
    DeviceState *d = nullptr;
    st = current_device(&d);
    if (st != CR_OK)
        return st;
    return launched(cr::qz::launch_quantize(w_rot, codebook, N, (int)K, qdata, srel, s_channel, d->num_sms, stream));
}

cr_status cr_w4a8_assign_codes(const float *w_rot, const uint8_t *srel, const float *s_channel, const float *codebook,
                               const float *rand, int64_t N, int64_t K, uint8_t *qdata, cr_stream_t stream)
{
    cr_status st = check_quant(w_rot, codebook, N, K, srel, s_channel, qdata);
    if (st != CR_OK || N == 0)
        return st;
    if (rand && !aligned16(rand))
        return CR_ERR_ALIGNMENT;
    DeviceState *d = nullptr;
    st = current_device(&d);
    if (st != CR_OK)
        return st;
    return launched(
        cr::qz::launch_assign(w_rot, srel, s_channel, codebook, rand, N, (int)K, qdata, d->num_sms, stream));
}

cr_status cr_w4a8_plan_create(const uint8_t *qdata, const uint8_t *srel, const float *codebook,
                              const float *s_channel, const float *bias, int64_t N, int64_t K, int act_qmax,
                              cr_out_dtype out_dtype, cr_w4a8_plan *plan)
{
    if (!plan)
        return CR_ERR_INVALID_ARG;
    *plan = nullptr;
    if (N < 0 || K < 0 || act_qmax < 1 || act_qmax > 127)
        return CR_ERR_INVALID_ARG;
    if (out_dtype != CR_OUT_BF16 && out_dtype != CR_OUT_F32)
        return CR_ERR_INVALID_ARG;
    cr_status st = check_k(K);
    if (st != CR_OK)
        return st;
    if (N > INT_MAX)
        return CR_ERR_UNSUPPORTED;
    if (N > 0) {
        if (!qdata || !srel || !codebook || !s_channel)
            return CR_ERR_INVALID_ARG;
        if (!aligned16(qdata) || !aligned16(srel) || !aligned16(codebook) || !aligned16(s_channel) ||
            (bias && !aligned16(bias)))
            return CR_ERR_ALIGNMENT;
    }
    DeviceState *d = nullptr;
    st = current_device(&d);
    if (st != CR_OK)
        return st;
    cr_w4a8_plan_st *p = new (std::nothrow) cr_w4a8_plan_st;
    if (!p)
        return CR_ERR_CUDA;
    cudaGetDevice(&p->device);
    p->d = d;
    p->qdata = qdata;
    p->srel = srel;
    p->codebook = codebook;
    p->s_channel = s_channel;
    p->bias = bias;
    p->N = N;
    p->K = K;
    p->act_qmax = act_qmax;
    p->out_dtype = out_dtype;
    if (N > 0) {
        cr_w4a8_layer ly{qdata, srel, s_channel, bias, N, nullptr, nullptr};
        st = build_gemv_args<1>(p->gemv, codebook, K, &ly, 1, out_dtype, 0, p->tiles, gemv_tile_rows(N, d->num_sms));
        if (st == CR_OK)
            st = check_split(*d, srel, codebook, N, K, p->split_ok);
        if (st != CR_OK) {
            delete p;
            return st;
        }
    }
    *plan = p;
    return CR_OK;
}

cr_status cr_w4a8_plan_destroy(cr_w4a8_plan plan)
{
    delete plan;
    return CR_OK;
}

cr_status cr_w4a8_plan_forward(cr_w4a8_plan plan, const uint16_t *x, int64_t M, void *out, int8_t *xq_work,
                               float *xs_work, cr_stream_t stream)
{
    if (!plan || M < 0)
        return CR_ERR_INVALID_ARG;
    if (M > INT_MAX)
        return CR_ERR_UNSUPPORTED;
    if (M == 0 || plan->N == 0)
        return CR_OK;
    if (!x || !out || !xq_work || !xs_work)
        return CR_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(out) || !aligned16(xq_work) || !aligned16(xs_work))
        return CR_ERR_ALIGNMENT;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev != plan->device) {
        cudaGetLastError();
        return CR_ERR_INVALID_ARG;
    }
    if (M > CR_GEMV_MAX_M)
        return linear_impl(x, plan->qdata, plan->srel, plan->codebook, plan->s_channel, plan->bias, M, plan->N,
                           plan->K, plan->act_qmax, plan->out_dtype, out, xq_work, xs_work, stream, 0);
    int64_t MP = 1;
    while (MP < M)
        MP <<= 1;
    cr_status st = launched(cr::rq::launch(x, M, plan->K, MP, plan->act_qmax, xq_work, xs_work, stream));
    if (st != CR_OK)
        return st;
    cr::gv::GemvArgs<1> args;
    {
        std::lock_guard<std::mutex> lock(plan->mu);
        if (plan->xmap_base != xq_work || plan->xmap_M != M) {
            if (!encode_gemv_x_map(&plan->gemv.tm_x, xq_work, M, plan->K))
                return CR_ERR_CUDA;
            plan->xmap_base = xq_work;
            plan->xmap_M = M;
        }
        args = plan->gemv;
    }
    args.xs = xs_work;
    args.M = (int)M;
    args.layer[0].out = out;
    return launch_gemv_args<1>(plan->d->num_sms, plan->d->gemv_attr_set, args, stream, /*pdl=*/true,
                               plan->split_ok, &plan->d->gemv_split_attr_set, &plan->d->gemv32_attr_set,
                               &plan->d->gemv32_split_attr_set);
}

cr_status cr_w4a8_plan_gemv(cr_w4a8_plan plan, const int8_t *xq, const float *xs, int64_t M, void *out,
                            cr_stream_t stream)
{
    if (!plan || M < 0)
        return CR_ERR_INVALID_ARG;
    if (M > CR_GEMV_MAX_M)
        return CR_ERR_UNSUPPORTED;
    if (M == 0 || plan->N == 0)
        return CR_OK;
    if (!xq || !xs || !out)
        return CR_ERR_INVALID_ARG;
    if (!aligned16(xq) || !aligned16(xs) || !aligned16(out))
        return CR_ERR_ALIGNMENT;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev != plan->device) {
        cudaGetLastError();
        return CR_ERR_INVALID_ARG;
    }
    cr::gv::GemvArgs<1> args;
    {
        std::lock_guard<std::mutex> lock(plan->mu);
        if (plan->xmap_base != xq || plan->xmap_M != M) {
            if (!encode_gemv_x_map(&plan->gemv.tm_x, xq, M, plan->K))
                return CR_ERR_CUDA;
            plan->xmap_base = xq;
            plan->xmap_M = M;
        }
        args = plan->gemv;
    }
    args.xs = xs;
    args.M = (int)M;
    args.layer[0].out = out;
    return launch_gemv_args<1>(plan->d->num_sms, plan->d->gemv_attr_set, args, stream, /*pdl=*/true,
                               plan->split_ok, &plan->d->gemv_split_attr_set, &plan->d->gemv32_attr_set,
                               &plan->d->gemv32_split_attr_set);
}

cr_status cr_w4a8_plan_forward_host(cr_w4a8_plan plan, const uint16_t *x_host, int64_t M, void *out_host,
                                    uint16_t *x_dev, void *out_dev, int8_t *xq_work, float *xs_work,
                                    cr_stream_t stream)
{
    if (!plan || M < 0)
        return CR_ERR_INVALID_ARG;
    if (M == 0 || plan->N == 0)
        return CR_OK;
    if (!x_host || !out_host)
        return CR_ERR_INVALID_ARG;
    const size_t xb = (size_t)(M * plan->K) * 2;
    const size_t ob = (size_t)(M * plan->N) * (plan->out_dtype == CR_OUT_F32 ? 4 : 2);
    // everything the forward checks, checked before the first copy is queued
    if (!x_dev || !out_dev || !xq_work || !xs_work)
        return CR_ERR_INVALID_ARG;
    if (!aligned16(x_dev) || !aligned16(out_dev) || !aligned16(xq_work) || !aligned16(xs_work))
        return CR_ERR_ALIGNMENT;
    if (M > INT_MAX)
        return CR_ERR_UNSUPPORTED;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev != plan->device) {
        cudaGetLastError();
        return CR_ERR_INVALID_ARG;
    }
    DeviceState *d = nullptr;
    cr_status st = current_device(&d);
    if (st != CR_OK)
        return st;
    // Small transfers between mapped page-locked host memory and the device
    // go through the SMs (ew::host_copy_kernel), anything else through the
    // copy engine.
    const void *x_map = small_mapped_host(x_host, xb);
    void *out_map = const_cast<void *>(small_mapped_host(out_host, ob));
    if (x_map) {
        st = launched(cr::ew::launch_host_copy(x_dev, x_map, (int64_t)xb, true, d->num_sms, stream));
        if (st != CR_OK)
            return st;
    } else if (cudaMemcpyAsync(x_dev, x_host, xb, cudaMemcpyHostToDevice, stream) != cudaSuccess) {
        cudaGetLastError();
        return CR_ERR_CUDA;
    }
    // A decode batch's GEMV stores y into mapped host memory itself: its
    // epilogue only stores the outputs, so the transfer is spread over the
    // launch instead of following it as another kernel.
    if (out_map && gemv_stores_host(plan, M))
        return cr_w4a8_plan_forward(plan, x_dev, M, out_map, xq_work, xs_work, stream);
    st = cr_w4a8_plan_forward(plan, x_dev, M, out_dev, xq_work, xs_work, stream);
    if (st != CR_OK)
        return st;
    if (out_map)
        return launched(cr::ew::launch_host_copy(out_map, out_dev, (int64_t)ob, false, d->num_sms, stream));
    if (cudaMemcpyAsync(out_host, out_dev, ob, cudaMemcpyDeviceToHost, stream) != cudaSuccess) {
        cudaGetLastError();
        return CR_ERR_CUDA;
    }
    return CR_OK;
}

cr_status cr_w4a8_plan_bind_host(cr_w4a8_plan plan, const uint16_t *x_host, int64_t M, void *out_host,
                                 uint16_t *x_dev, void *out_dev, int8_t *xq_work, float *xs_work,
                                 cr_w4a8_host_call *call)
{
    if (!call)
        return CR_ERR_INVALID_ARG;
    *call = nullptr;
    if (!plan || M < 0)
        return CR_ERR_INVALID_ARG;
    if (M > INT_MAX)
        return CR_ERR_UNSUPPORTED;
    cr_w4a8_host_call_st *c = new (std::nothrow) cr_w4a8_host_call_st();
    if (!c)
        return CR_ERR_CUDA;
    c->plan = plan;
    c->M = M;
    if (M > 0 && plan->N > 0) {
        cr_status st = CR_OK;
        int dev = -1;
        if (!x_host || !out_host || !x_dev || !out_dev || !xq_work || !xs_work)
            st = CR_ERR_INVALID_ARG;
        else if (!aligned16(x_dev) || !aligned16(out_dev) || !aligned16(xq_work) || !aligned16(xs_work))
            st = CR_ERR_ALIGNMENT;
        else if (cudaGetDevice(&dev) != cudaSuccess || dev != plan->device) {
            cudaGetLastError();
            st = CR_ERR_INVALID_ARG;
        }
        if (st == CR_OK && M <= CR_GEMV_MAX_M) {
            std::lock_guard<std::mutex> lock(plan->mu);
            c->gemv = plan->gemv;
            if (!encode_gemv_x_map(&c->gemv.tm_x, xq_work, M, plan->K))
                st = CR_ERR_CUDA;
        }
        if (st != CR_OK) {
            delete c;
            return st;
        }
        c->x_host = x_host;
        c->out_host = out_host;
        c->x_dev = x_dev;
        c->out_dev = out_dev;
        c->xq = xq_work;
        c->xs = xs_work;
        c->xb = (size_t)(M * plan->K) * 2;
        c->ob = (size_t)(M * plan->N) * (plan->out_dtype == CR_OUT_F32 ? 4 : 2);
        c->x_map = small_mapped_host(x_host, c->xb);
        c->out_map = const_cast<void *>(small_mapped_host(out_host, c->ob));
        c->MP = 1;
        while (c->MP < M)
            c->MP <<= 1;
        c->gemv.xs = xs_work;
        c->gemv.M = (int)M;
        // as in cr_w4a8_plan_forward_host
        c->gemv.layer[0].out = (c->out_map && gemv_stores_host(plan, M)) ? c->out_map : out_dev;
    }
    *call = c;
    return CR_OK;
}

cr_status cr_w4a8_host_call_run(cr_w4a8_host_call c, cr_stream_t stream)
{
    if (!c)
        return CR_ERR_INVALID_ARG;
    cr_w4a8_plan plan = c->plan;
    if (c->M == 0 || plan->N == 0)
        return CR_OK;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev != plan->device) {
        cudaGetLastError();
        return CR_ERR_INVALID_ARG;
    }
    DeviceState *d = plan->d;
    cr_status st = CR_OK;
    if (c->x_map)
        st = launched(cr::ew::launch_host_copy(c->x_dev, c->x_map, (int64_t)c->xb, true, d->num_sms, stream));
    else if (cudaMemcpyAsync(c->x_dev, c->x_host, c->xb, cudaMemcpyHostToDevice, stream) != cudaSuccess) {
        cudaGetLastError();
        st = CR_ERR_CUDA;
    }
    if (st != CR_OK)
        return st;
    if (c->M > CR_GEMV_MAX_M) {
        st = cr_w4a8_plan_forward(plan, c->x_dev, c->M, c->out_dev, c->xq, c->xs, stream);
    } else {
        st = launched(cr::rq::launch(c->x_dev, c->M, plan->K, c->MP, plan->act_qmax, c->xq, c->xs, stream));
        if (st == CR_OK)
            st = launch_gemv_args<1>(d->num_sms, d->gemv_attr_set, c->gemv, stream, /*pdl=*/true, plan->split_ok,
                                     &d->gemv_split_attr_set, &d->gemv32_attr_set, &d->gemv32_split_attr_set);
    }
    if (st != CR_OK)
        return st;
    if (c->out_map && gemv_stores_host(plan, c->M))
        return CR_OK;  // the GEMV stored y into out_host
    if (c->out_map)
        return launched(cr::ew::launch_host_copy(c->out_map, c->out_dev, (int64_t)c->ob, false, d->num_sms, stream));
    if (cudaMemcpyAsync(c->out_host, c->out_dev, c->ob, cudaMemcpyDeviceToHost, stream) != cudaSuccess) {
        cudaGetLastError();
        return CR_ERR_CUDA;
    }
    return CR_OK;
}

cr_status cr_w4a8_host_call_destroy(cr_w4a8_host_call call)
{
    delete call;
    return CR_OK;
}

cr_status cr_interleave_rows(const void *src, void *dst, int64_t rows, int64_t row_bytes, cr_stream_t stream)
{
    if (rows < 0 || row_bytes < 0 || rows % 2 != 0)
        return CR_ERR_INVALID_ARG;
    if (rows == 0 || row_bytes == 0)
        return CR_OK;
    if (!src || !dst || rows > INT64_MAX / row_bytes)
        return CR_ERR_INVALID_ARG;
    const uintptr_t s0 = (uintptr_t)src, d0 = (uintptr_t)dst, n = (uintptr_t)(rows * row_bytes);
    if (s0 < d0 + n && d0 < s0 + n)
        return CR_ERR_INVALID_ARG;  // the copy is not in place
    DeviceState *d = nullptr;
    const cr_status st = current_device(&d);
    if (st != CR_OK)
        return st;
    return launched(cr::ew::launch_interleave_rows(src, dst, rows, row_bytes, d->num_sms, stream));
}

cr_status cr_w4a8_gemv_grouped(const int8_t *xq, const float *xs, const float *codebook, int64_t M, int64_t K,
                               const cr_w4a8_layer *layers, int num_layers, cr_out_dtype out_dtype,
                               cr_stream_t stream)
{
    if (M > CR_GEMV_MAX_M)
        return CR_ERR_UNSUPPORTED;
    cr_status st = check_layers(xq, xs, codebook, M, K, layers, num_layers, out_dtype, /*allow_acc=*/true);
    if (st != CR_OK || M == 0 || total_rows(layers, num_layers) == 0)
        return st;
    DeviceState *d = nullptr;
    st = current_device(&d);
    if (st != CR_OK)
        return st;
    return run_gemv_layers(*d, xq, xs, codebook, M, K, layers, num_layers, out_dtype,
                           stream, /*pdl=*/true);
}

cr_status cr_w4a8_linear_grouped(const uint16_t *x, const float *codebook, int64_t M, int64_t K,
                                 const cr_w4a8_layer *layers, int num_layers, int act_qmax,
                                 cr_out_dtype out_dtype, int8_t *xq_work, float *xs_work, cr_stream_t stream)
{
    if (M < 0 || K < 0 || act_qmax < 1 || act_qmax > 127)
        return CR_ERR_INVALID_ARG;
    int64_t MP = M;
    if (M >= 1 && M <= CR_GEMV_MAX_M) {
        MP = 1;
        while (MP < M)
            MP <<= 1;
    }
    cr_status st = check_layers(xq_work, xs_work, codebook, M, K, layers, num_layers, out_dtype,
                                /*allow_acc=*/false);
    if (st != CR_OK || M == 0 || total_rows(layers, num_layers) == 0)
        return st;
    if (!x)
        return CR_ERR_INVALID_ARG;
    if (!aligned16(x))
        return CR_ERR_ALIGNMENT;
    DeviceState *d = nullptr;
    st = current_device(&d);
    if (st != CR_OK)
        return st;
    auto activations = [&]() { return launched(cr::rq::launch(x, M, K, MP, act_qmax, xq_work, xs_work, stream)); };
    if (M <= CR_GEMV_MAX_M) {
        st = activations();
        if (st != CR_OK)
            return st;
        return run_gemv_layers(*d, xq_work, xs_work, codebook, M, K, layers, num_layers,
                               out_dtype, stream, /*pdl=*/true);
    }
    // the first layer's weight decode overlaps the activation kernel
    const std::function<cr_status()> act = activations;
    bool first = true;
    for (int l = 0; l < num_layers; ++l) {
        const cr_w4a8_layer &ly = layers[l];
        if (ly.N == 0)
            continue;
        st = run_gemm(*d, xq_work, xs_work, ly.qdata, ly.srel, codebook, ly.s_channel, ly.bias, M, ly.N, K, out_dtype,
                      ly.out, nullptr, stream, first ? &act : nullptr);
        if (st != CR_OK)
            return st;
        first = false;
    }
    return CR_OK;
}

// ---------------------------------------------------------------- decode forward without allocation
//
// The scratch of cr_w4a8_linear_decode_noalloc: the padded int8 activations
// (at most 8 rows of K <= CR_MAX_K bytes) at offset 0 and their 8 fp32 scales
// at offset CR_GEMV_MAX_M * CR_MAX_K.  One array per device, reserved when the
// module loads on that device.  In host code `g_noalloc_scratch` is only a
// host-side stand-in for the symbol: its device address is looked up once per
// device with cudaGetSymbolAddress and that address is what the kernels get.
static __device__ __align__(256) uint8_t g_noalloc_scratch[CR_NOALLOC_SCRATCH_BYTES];

namespace {
struct NoallocState {
    bool ready = false;
    uint8_t *scratch = nullptr;  // device address of g_noalloc_scratch on this device
    int num_sms = 0;
    std::atomic<bool> gemv_attr_set{false};  // set in noalloc_scratch, under the lock
};
NoallocState g_noalloc[kMaxDevices];

// Once per device, with that device current: check it is an sm_100 part,
// look up the scratch array's device address, the SM count and the tensor-map
// encoder, and set the decode GEMV's shared-memory attribute.  Allocates
// nothing.
cr_status noalloc_scratch(NoallocState **out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return CR_ERR_NO_DEVICE;
    }
    std::lock_guard<std::mutex> lock(g_mutex);
    NoallocState &s = g_noalloc[dev];
    if (!s.ready) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
            cudaGetLastError();
            return CR_ERR_NO_DEVICE;
        }
        if (major != 10 || minor != 0)
            return CR_ERR_NO_DEVICE;
        if (cudaDeviceGetAttribute(&s.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            cudaGetLastError();
            return CR_ERR_NO_DEVICE;
        }
        if (!have_encode_tiled())
            return CR_ERR_NO_DEVICE;
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return CR_ERR_CUDA;
        }
        s.scratch = static_cast<uint8_t *>(p);
        if (cudaFuncSetAttribute(cr::gv::gemv_kernel<cr::gv::Prod, 1, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)cr::gv::Prod::kSmemBytes) != cudaSuccess ||
            cr::rq::set_attributes() != cudaSuccess) {
            cudaGetLastError();
            return CR_ERR_CUDA;
        }
        s.gemv_attr_set = true;
        s.ready = true;
    }
    *out = &s;
    return CR_OK;
}
}  // namespace

cr_status cr_w4a8_linear_decode_noalloc(const uint16_t *x, const uint8_t *qdata, const uint8_t *srel,
                                        const float *codebook, const float *s_channel, const float *bias,
                                        int64_t M, int64_t N, int64_t K, int act_qmax, cr_out_dtype out_dtype,
                                        void *out, cr_stream_t stream)
{
    if (M < 0 || N < 0 || K < 0 || act_qmax < 1 || act_qmax > 127 ||
        (out_dtype != CR_OUT_BF16 && out_dtype != CR_OUT_F32))
        return CR_ERR_INVALID_ARG;
    const cr_status k = check_k(K);
    if (k != CR_OK)
        return k;
    if (M > CR_GEMV_MAX_M)
        return CR_ERR_UNSUPPORTED;  // the padded activations would not fit the static scratch
    if (N > INT_MAX)
        return CR_ERR_UNSUPPORTED;
    if (M == 0 || N == 0)
        return CR_OK;
    int64_t MP = 1;
    while (MP < M)
        MP <<= 1;
    if (MP * K > (int64_t)CR_GEMV_MAX_M * CR_MAX_K)
        return CR_ERR_UNSUPPORTED;
    if (!x || !qdata || !srel || !codebook || !s_channel || !out)
        return CR_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(qdata) || !aligned16(srel) || !aligned16(codebook) || !aligned16(s_channel) ||
        !aligned16(out) || (bias && !aligned16(bias)))
        return CR_ERR_ALIGNMENT;
    NoallocState *ns = nullptr;
    const cr_status ss = noalloc_scratch(&ns);
    if (ss != CR_OK)
        return ss;
    int8_t *xq = reinterpret_cast<int8_t *>(ns->scratch);
    float *xs = reinterpret_cast<float *>(ns->scratch + (size_t)CR_GEMV_MAX_M * CR_MAX_K);
    // The activation kernel rewrites every scratch byte the GEMV reads (rows
    // M..MP-1 as zeros with scale 1), so nothing left by an earlier call leaks in.
    cr_status st = launched(cr::rq::launch(x, M, K, MP, act_qmax, xq, xs, stream));
    if (st != CR_OK)
        return st;
    return run_gemv(ns->num_sms, ns->gemv_attr_set, xq, xs, qdata, srel, codebook, s_channel, bias, M, N, K,
                    out_dtype, out, nullptr, stream, /*pdl=*/true);
}

cr_status cr_gemm_s8(const int8_t *xq, const float *xs, const int8_t *w8, const float *s_channel, const float *bias,
                     int64_t M, int64_t N, int64_t K, cr_out_dtype out_dtype, void *out, int32_t *acc_out,
                     cr_stream_t stream)
{
    if (M < 0 || N < 0 || K < 0)
        return CR_ERR_INVALID_ARG;
    if (out_dtype != CR_OUT_BF16 && out_dtype != CR_OUT_F32)
        return CR_ERR_INVALID_ARG;
    cr_status st = check_k(K);
    if (st != CR_OK)
        return st;
    if (M > INT_MAX || N > INT_MAX)
        return CR_ERR_UNSUPPORTED;
    if (M == 0 || N == 0)
        return CR_OK;
    if (!xq || !xs || !w8 || !s_channel || !out)
        return CR_ERR_INVALID_ARG;
    if (!aligned16(xq) || !aligned16(xs) || !aligned16(w8) || !aligned16(s_channel) || !aligned16(out) ||
        (bias && !aligned16(bias)) || (acc_out && !aligned16(acc_out)))
        return CR_ERR_ALIGNMENT;
    DeviceState *d = nullptr;
    st = current_device(&d);
    if (st != CR_OK)
        return st;
    return gemm_on_w8(*d, xq, xs, w8, s_channel, bias, M, N, K, out_dtype, out, acc_out, stream, 0);
}

cr_status cr_mma_i8_peak(int64_t iters, double *ops_per_launch, cr_stream_t stream)
{
    if (iters < 1 || iters > (1 << 20) || !ops_per_launch)
        return CR_ERR_INVALID_ARG;
    DeviceState *d = nullptr;
    const cr_status st = current_device(&d);
    if (st != CR_OK)
        return st;
    if (!d->peak_attr_set) {
        if (cudaFuncSetAttribute(cr::pk::mma_i8_peak_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)cr::pk::kSmemBytes) != cudaSuccess) {
            cudaGetLastError();
            return CR_ERR_CUDA;
        }
        d->peak_attr_set = true;
    }
    const int pairs = d->num_sms / 2;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(2 * pairs));
    cfg.blockDim = dim3(cr::pk::kThreads);
    cfg.dynamicSmemBytes = cr::pk::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    *ops_per_launch = 2.0 * 256.0 * 256.0 * 128.0 * (double)iters * (double)pairs;
    return launched(cudaLaunchKernelEx(&cfg, cr::pk::mma_i8_peak_kernel, (int)iters));
}

cr_status cr_selftest_wait_timeout(uint64_t limit_ns, cr_stream_t stream)
{
    if (limit_ns < 1000000ull || limit_ns > 1000000000ull)
        return CR_ERR_INVALID_ARG;
    DeviceState *d = nullptr;
    const cr_status st = current_device(&d);
    if (st != CR_OK)
        return st;
    cr::ew::selftest_timeout_kernel<<<1, 32, 0, stream>>>(limit_ns);
    return launched(cudaGetLastError());
}

cr_status cr_check_device_error(cr_stream_t stream)
{
    DeviceState *d = nullptr;
    const cr_status ds = current_device(&d);
    if (ds != CR_OK)
        return ds;
    if (cudaStreamSynchronize(stream) != cudaSuccess) {
        cudaGetLastError();
        return CR_ERR_CUDA;
    }
    int v = 0;
    const int zero = 0;
    if (cudaMemcpyFromSymbol(&v, cr::g_device_error, sizeof(int)) != cudaSuccess ||
        cudaMemcpyToSymbol(cr::g_device_error, &zero, sizeof(int)) != cudaSuccess) {
        cudaGetLastError();
        return CR_ERR_CUDA;
    }
    return v ? CR_ERR_TIMEOUT : CR_OK;
}

}  // extern "C"

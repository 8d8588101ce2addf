// Host side of the C ABI declared in include/awq.h: argument validation,
// workspace layout, TMA descriptor encoding and kernel launches.  Every step
// of the search runs in the kernels of awq_kernels.cuh; nothing here computes
// on the host beyond sizes and launch shapes.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "awq.h"
#include "awq_kernels.cuh"

namespace {

std::atomic<uint32_t> g_timeout_ms{4000};

// One-shot, per-thread request to bracket the next search kernel with events.
thread_local cudaEvent_t t_prof_begin = nullptr;
thread_local cudaEvent_t t_prof_end = nullptr;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_qcfg(const awq_qcfg &q) {
    return (q.bits == 2 || q.bits == 3 || q.bits == 4) && (q.group_size == 64 || q.group_size == 128) &&
           (q.zero_point == 0 || q.zero_point == 1);
}

constexpr int64_t kMaxDim = (int64_t(1) << 31) - 1;
constexpr int kMaxAlpha = 64;
constexpr int64_t kMaxGptqK = 8192;      // the GPTQ sweep keeps its rows and a ring of U rows on chip

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Workspace of awq_search_layer, carved in this order (each 256-byte aligned):
//   s_tab   float [n_alpha][K]
//   rs_tab  float [n_alpha][K]
//   params  uint2 [n_alpha][K/g][N_pad]   (N_pad = N rounded up to 256; padded rows are zero)
//   partial float [n_alpha][ceil(T/512)][N]
int64_t padded_rows(int64_t N) { return (N + awq::srch2::PM - 1) / awq::srch2::PM * awq::srch2::PM; }
struct SearchWs {
    size_t s_off, rs_off, prm_off, part_off, xm_off, total;
};
// masked: room for X with the fp16-kept channels zeroed, [T][K] fp16.
SearchWs search_ws_layout(int64_t N, int64_t K, int64_t T, int group, int n_alpha, bool masked = false) {
    SearchWs w{};
    const int64_t n_tb = (T + awq::srch2::BT - 1) / awq::srch2::BT;
    size_t off = 0;
    w.s_off = off;    off = round_up(off + sizeof(float) * (size_t)n_alpha * K, 256);
    w.rs_off = off;   off = round_up(off + sizeof(float) * (size_t)n_alpha * K, 256);
    w.prm_off = off;  off = round_up(off + sizeof(uint2) * (size_t)n_alpha * (K / group) * padded_rows(N), 256);
    w.part_off = off; off = round_up(off + sizeof(float) * (size_t)n_alpha * n_tb * N, 256);
    w.xm_off = off;   if (masked) off = round_up(off + 2 * (size_t)T * K, 256);
    w.total = off;
    return w;
}
// One pass of the tensor-core decode, launched so that it may start while the
// prep grid before it on the stream still runs (programmatic dependent launch):
// its code stream, tensor-memory allocation and barrier set-up overlap the prep,
// and the roles that read the prep's outputs wait for it (griddepcontrol.wait).
template <int NR, int CB, int GPS>
cudaError_t launch_qtc(unsigned grid, cudaStream_t st, const CUtensorMap &tmap_codes, const CUtensorMap &tmap_b,
                       const awq::qtc::Args &A) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(awq::qtc::THREADS);
    cfg.dynamicSmemBytes = awq::qtc::smem_bytes<NR>();
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, awq::qlinear_tc_kernel<NR, CB, GPS>, tmap_codes, tmap_b, A);
}

// The dynamic shared memory of the tensor-core decode instantiations.
template <int NR>
bool qtc_attrs() {
    const int b = (int)awq::qtc::smem_bytes<NR>();
    return cudaFuncSetAttribute(awq::qlinear_tc_kernel<NR, 4, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, b) ==
               cudaSuccess &&
           cudaFuncSetAttribute(awq::qlinear_tc_kernel<NR, 4, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize, b) ==
               cudaSuccess &&
           cudaFuncSetAttribute(awq::qlinear_tc_kernel<NR, 2, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, b) ==
               cudaSuccess &&
           cudaFuncSetAttribute(awq::qlinear_tc_kernel<NR, 2, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize, b) ==
               cudaSuccess;
}


awq_status cuda_status(cudaError_t e) { return e == cudaSuccess ? AWQ_OK : AWQ_ERR_CUDA; }

awq_status last_launch() { return cuda_status(cudaGetLastError()); }

// Per-device facts, queried once.
struct DevInfo {
    int sms = 0;
    int cc_major = 0;
    bool search_attr = false;
    int max_pairs = 0;       // CTA pairs of the search kernel that fit on the device at once
};
std::mutex g_dev_mu;
DevInfo g_dev[64];

awq_status device_info(DevInfo &out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return AWQ_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_dev_mu);
    DevInfo &d = g_dev[dev];
    if (d.sms == 0) {
        if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
            d.sms = 0;
            return AWQ_ERR_CUDA;
        }
    }
    if (d.cc_major != 10) return AWQ_ERR_UNSUPPORTED;
    if (!d.search_attr) {
        if (cudaFuncSetAttribute(awq::srch2::search_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)awq::srch2::SMEM_BYTES) != cudaSuccess)
            return AWQ_ERR_CUDA;
        // A pair must sit in one GPC, so fewer than sms/2 pairs may fit at once;
        // the persistent grid never exceeds what is co-resident.
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * (d.sms / 2), 1, 1);
        cfg.blockDim = dim3(awq::srch2::NUM_THREADS, 1, 1);
        cfg.dynamicSmemBytes = awq::srch2::SMEM_BYTES;
        int clusters = 0;
        if (cudaOccupancyMaxActiveClusters(&clusters, (void *)awq::srch2::search_pair_kernel, &cfg) != cudaSuccess ||
            clusters <= 0) {
            (void)cudaGetLastError();
            clusters = d.sms / 2;
        }
        d.max_pairs = clusters < d.sms / 2 ? clusters : d.sms / 2;
        if (cudaFuncSetAttribute(awq::qlinear_gemv_kernel<4, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 awq::qlv::SMEM_LIMIT) != cudaSuccess ||
            cudaFuncSetAttribute(awq::qlinear_gemv_kernel<4, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 awq::qlv::SMEM_LIMIT) != cudaSuccess ||
            cudaFuncSetAttribute(awq::qlinear_gemv_kernel<2, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 awq::qlv::SMEM_LIMIT) != cudaSuccess ||
            cudaFuncSetAttribute(awq::qlinear_gemv_kernel<2, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 awq::qlv::SMEM_LIMIT) != cudaSuccess ||
            cudaFuncSetAttribute(awq::qlinear_gemv_kernel<4, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 awq::qlv::SMEM_LIMIT) != cudaSuccess ||
            !qtc_attrs<16>() || !qtc_attrs<32>() || !qtc_attrs<48>() ||
            cudaFuncSetAttribute(awq::gptq_hessian_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)awq::ghs::SMEM_BYTES) != cudaSuccess ||
            cudaFuncSetAttribute(awq::gptq_sweep_kernel<1, 8, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 awq::qlv::SMEM_LIMIT) != cudaSuccess ||
            cudaFuncSetAttribute(awq::gptq_sweep_kernel<2, 8, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 awq::qlv::SMEM_LIMIT) != cudaSuccess ||
            cudaFuncSetAttribute(awq::gptq_sweep_kernel<4, 8, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 awq::qlv::SMEM_LIMIT) != cudaSuccess ||
            cudaFuncSetAttribute(awq::gptq_sweep_kernel<8, 8, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 awq::qlv::SMEM_LIMIT) != cudaSuccess ||
            cudaFuncSetAttribute(awq::gptq_sweep_kernel<16, 4, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 awq::qlv::SMEM_LIMIT) != cudaSuccess)
            return AWQ_ERR_CUDA;
        d.search_attr = true;
    }
    out = d;
    return AWQ_OK;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda).
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// A row-major fp16 matrix [rows, ld] as a 2-D tensor (inner dimension
// `cols`), boxes of 64 columns x box_rows rows, 128-byte swizzle; rows past the
// end read as zeros.
bool encode_rows_map(CUtensorMap *m, const void *base, int64_t rows, int64_t cols, int64_t ld, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
    cuuint32_t box[2] = {(cuuint32_t)awq::srch2::BK, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Packed codes [rows][words] (uint32) as a 2-D tensor, boxes of
// qlv::WORDS words x qlv::ROWS rows, no swizzle; rows and words past the end
// read as zeros.
bool encode_codes_map(CUtensorMap *m, const uint32_t *codes, int64_t rows, int64_t words) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)words, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)words * 4};
    cuuint32_t box[2] = {(cuuint32_t)awq::qlv::WORDS, (cuuint32_t)awq::qlv::ROWS};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t *>(codes), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Packed code words [rows][words] as boxes of box_words x box_rows: 32 words
// (128 bytes) with the 128-byte swizzle, 16 words (64 bytes) with the 64-byte one.
bool encode_words_map(CUtensorMap *m, const uint32_t *codes, int64_t rows, int64_t words, int box_words,
                      int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)words, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)words * 4};
    cuuint32_t box[2] = {(cuuint32_t)box_words, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t *>(codes), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE,
                    box_words == 32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}
// bf16 [rows][cols] as boxes of 64 columns x box_rows rows, 128-byte swizzle.
bool encode_bf16_map(CUtensorMap *m, const void *base, int64_t rows, int64_t cols, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int blocks_for(int64_t threads_total, int block) {
    int64_t b = (threads_total + block - 1) / block;
    return (int)(b < 1 ? 1 : b);
}

awq_status launch_group_params(const void *W, int64_t N, int64_t K, awq_qcfg q, const float *s_tab,
                               int n_alpha, const uint8_t *mask, uint2 *params, cudaStream_t st) {
    const int group = q.group_size;
    const float qmax = (float)((1 << q.bits) - 1);
    const int sym = q.zero_point ? 0 : 1;
    const int G = (int)(K / group);
    const int lpr = group / awq::kGpCols;
    const int64_t N_pad = padded_rows(N);
    const int64_t rows_per_block = awq::kGpThreads / lpr;
    const int64_t row_blocks = (N_pad + rows_per_block - 1) / rows_per_block;
    const size_t smem = sizeof(float) * (size_t)n_alpha * lpr * (awq::kGpCols + 4);
    const unsigned grid = (unsigned)(row_blocks * G);
    if (lpr == 2)
        awq::group_params_kernel<2><<<grid, awq::kGpThreads, smem, st>>>((const __half *)W, N, N_pad, K, G, s_tab,
                                                                        n_alpha, qmax, sym, mask, params);
    else
        awq::group_params_kernel<1><<<grid, awq::kGpThreads, smem, st>>>((const __half *)W, N, N_pad, K, G, s_tab,
                                                                        n_alpha, qmax, sym, mask, params);
    return last_launch();
}

// Scratch for awq_search_layer_noalloc: lives in the library's device image,
// so no allocation happens at call time.  In host code `g_noalloc_scratch` is
// only a stand-in symbol, never a device address: the address is looked up
// once per device with cudaGetSymbolAddress and cached.
static __device__ __align__(256) uint8_t g_noalloc_scratch[AWQ_NOALLOC_SCRATCH_BYTES];
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[64] = {};

awq_status noalloc_scratch(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return AWQ_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return AWQ_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return AWQ_OK;
}

// Workspace of awq_qlinear: x' = x / s as binary32 [T_pad][Kp] in the decode
// kernel's stage order (T rounded up to the tokens of one pass, K to the
// widest stage), the partial sums of row blocks split across blocks, and the
// per row block arrival counters.
constexpr int64_t kQlMaxGrid = 1024;
constexpr int64_t kQlTcMinTokens = 2;      // awq_qlinear: tensor cores from 2 tokens on
int64_t ql_rows_pad(int64_t T) { return (T + awq::qlv::TOKENS - 1) / awq::qlv::TOKENS * awq::qlv::TOKENS; }
int64_t ql_cols_pad(int64_t K, int64_t sc) { return (K + sc - 1) / sc * sc; }
size_t ql_xs_bytes(int64_t T, int64_t K) {
    return round_up(sizeof(float) * (size_t)ql_rows_pad(T) * ql_cols_pad(K, awq::qlv::MAX_STAGE_COLS), 256);
}
int64_t ql_row_blocks(int64_t N) { return (N + awq::qlv::ROWS - 1) / awq::qlv::ROWS; }
size_t ql_part_bytes(int64_t N) {
    return round_up(sizeof(float) * (size_t)(ql_row_blocks(N) + kQlMaxGrid) * awq::qlv::SLOT_FLOATS, 256);
}
size_t qlinear_ws_simt(int64_t T, int64_t K, int64_t N) {
    return ql_xs_bytes(T, K) + ql_part_bytes(N) +
           round_up(sizeof(unsigned) * (size_t)ql_row_blocks(N) * awq::qlv::RGROUPS, 256);
}
// The tensor-core path: x' pieces bf16 [passes][NR][Kp], group sums fp32
// [passes][K/64 or fewer groups][16], partial sums of row blocks split across
// blocks fp32 [(row blocks + grid) * 128][16] and their arrival counters.
struct QtcPlan {
    int NR, TT, n_pass;
    int64_t Kp, row_blocks, n_steps, units;
    size_t xb_bytes, gs_bytes, part_bytes, cnt_bytes;
};
QtcPlan qtc_plan(int64_t T, int64_t K, int64_t N, int group) {
    QtcPlan p;
    p.NR = T <= 5 ? 16 : T <= 10 ? 32 : 48;
    p.TT = awq::qtc::tile_tokens(p.NR);
    p.n_pass = (int)((T + p.TT - 1) / p.TT);
    p.Kp = (K + 63) / 64 * 64;
    p.row_blocks = (N + awq::qtc::ROWS - 1) / awq::qtc::ROWS;
    p.n_steps = (K + awq::qtc::SC - 1) / awq::qtc::SC;
    p.units = p.row_blocks * p.n_steps;
    p.xb_bytes = round_up(2 * (size_t)p.n_pass * p.NR * p.Kp, 1024);
    p.gs_bytes = round_up(4 * (size_t)p.n_pass * (size_t)(K / group) * 16, 256);
    p.part_bytes = round_up(sizeof(float) * (size_t)(p.row_blocks + kQlMaxGrid) * awq::qtc::SLOT_FLOATS, 256);
    p.cnt_bytes = round_up(sizeof(unsigned) * (size_t)p.row_blocks * 4, 256);
    return p;
}
size_t qtc_ws_bound(int64_t T, int64_t K, int64_t N) {
    // the largest plan over group sizes: 64-column groups
    const QtcPlan p = qtc_plan(T, K, N, 64);
    return p.xb_bytes + p.gs_bytes + p.part_bytes + p.cnt_bytes;
}
size_t qlinear_ws(int64_t T, int64_t K, int64_t N) {
    const size_t a = qlinear_ws_simt(T, K, N), b = qtc_ws_bound(T, K, N);
    return a > b ? a : b;
}

// a8 for a given s: codes, fp16 scales and zeros.
awq_status launch_pack(const void *W, int64_t N, int64_t K, const float *s, awq_qcfg q, uint32_t *codes,
                       void *scales, void *zeros, cudaStream_t st) {
    DevInfo d;
    if (awq_status e = device_info(d)) return e;
    const int G = (int)(K / q.group_size);
    const int sym = q.zero_point ? 0 : 1;
    // one warp per item of 4 rows x 256 columns, at most 8 blocks per SM (the rest loop)
    const int64_t items = (N + awq::kPkRows - 1) / awq::kPkRows * ((K + awq::kPkCols - 1) / awq::kPkCols);
    const int64_t warps_per_block = awq::kPkThreads / 32;
    int64_t grid = (items + warps_per_block - 1) / warps_per_block;
    if (grid > 8 * (int64_t)d.sms) grid = 8 * (int64_t)d.sms;
    if (q.group_size == 128)
        awq::pack_kernel<16><<<(unsigned)grid, awq::kPkThreads, 0, st>>>((const __half *)W, N, K, G, q.bits, sym, s,
                                                                        codes, (__half *)scales, (__half *)zeros);
    else
        awq::pack_kernel<8><<<(unsigned)grid, awq::kPkThreads, 0, st>>>((const __half *)W, N, K, G, q.bits, sym, s,
                                                                       codes, (__half *)scales, (__half *)zeros);
    return last_launch();
}

// a3-a6 on tables of n scale vectors already in the workspace: group
// parameters, the tensor-core search against X, the loss reduction.
awq_status run_search(const void *W, int64_t N, int64_t K, const void *X, int64_t T, int64_t ldx, int group,
                      float qmax, const float *s_tab, const float *rs_tab, int n_alpha, const uint2 *params,
                      float *partial, float *losses, float *row_losses, int64_t norm_rows, const DevInfo &d,
                      cudaStream_t st);

awq_status search_core(const void *W, int64_t N, int64_t K, const void *X, int64_t T, int64_t ldx, awq_qcfg q,
                       const float *s_tab, const float *rs_tab, int n_alpha, const uint8_t *mask, uint2 *params,
                       float *partial, float *losses, float *row_losses, int64_t norm_rows, const DevInfo &d,
                       cudaStream_t st) {
    // a3 (group parameters for every alpha)
    if (awq_status e = launch_group_params(W, N, K, q, s_tab, n_alpha, mask, params, st)) return e;
    return run_search(W, N, K, X, T, ldx, q.group_size, (float)((1 << q.bits) - 1), s_tab, rs_tab, n_alpha, params,
                      partial, losses, row_losses, norm_rows, d, st);
}

// a4-a6 with the group parameters already in the workspace.
awq_status run_search(const void *W, int64_t N, int64_t K, const void *X, int64_t T, int64_t ldx, int group,
                      float qmax, const float *s_tab, const float *rs_tab, int n_alpha, const uint2 *params,
                      float *partial, float *losses, float *row_losses, int64_t norm_rows, const DevInfo &d,
                      cudaStream_t st) {
    // a4-a6: the tensor-core search on CTA pairs
    CUtensorMap tmap_x, tmap_w;
    if (!encode_rows_map(&tmap_x, X, T, K, ldx, awq::srch2::HN) ||
        !encode_rows_map(&tmap_w, W, N, K, K, awq::srch2::BM))
        return AWQ_ERR_CUDA;
    awq::srch2::Args A;
    A.params = params;
    A.s_tab = s_tab;
    A.rs_tab = rs_tab;
    A.partial = partial;
    A.N = N;
    A.K = K;
    A.T = T;
    A.N_pad = padded_rows(N);
    A.n_alpha = n_alpha;
    A.G = (int)(K / group);
    A.group = group;
    A.n_tb = (int)((T + awq::srch2::BT - 1) / awq::srch2::BT);
    A.n_kb = (int)(K / awq::srch2::BK);
    A.n_units = (A.N_pad / awq::srch2::PM) * A.n_tb * n_alpha;
    A.qmax = qmax;
    A.timeout_ns = (uint64_t)g_timeout_ms.load() * 1000000ull;
    const int64_t pairs = A.n_units < d.max_pairs ? A.n_units : d.max_pairs;
    const int grid = (int)(2 * pairs);
    cudaEvent_t pb = t_prof_begin, pe = t_prof_end;
    t_prof_begin = t_prof_end = nullptr;
    if (pb && cudaEventRecord(pb, st) != cudaSuccess) return AWQ_ERR_CUDA;
    awq::srch2::search_pair_kernel<<<grid, awq::srch2::NUM_THREADS, awq::srch2::SMEM_BYTES, st>>>(tmap_x, tmap_w, A);
    if (awq_status e = last_launch()) return e;
    if (pe && cudaEventRecord(pe, st) != cudaSuccess) return AWQ_ERR_CUDA;

    // a6: deterministic reduction to per-alpha MSE (and optional per-row sums)
    awq::loss_reduce_kernel<<<n_alpha, awq::kLossThreads, 0, st>>>(partial, N, T, A.n_tb, norm_rows, losses,
                                                                   row_losses);
    return last_launch();
}

}  // namespace

extern "C" {

const char *awq_status_string(awq_status s) {
    switch (s) {
        case AWQ_OK: return "AWQ_OK";
        case AWQ_ERR_INVALID_ARG: return "AWQ_ERR_INVALID_ARG";
        case AWQ_ERR_UNSUPPORTED: return "AWQ_ERR_UNSUPPORTED";
        case AWQ_ERR_CUDA: return "AWQ_ERR_CUDA";
        case AWQ_ERR_TIMEOUT: return "AWQ_ERR_TIMEOUT";
        case AWQ_ERR_WORKSPACE: return "AWQ_ERR_WORKSPACE";
    }
    return "AWQ_ERR_UNKNOWN";
}

void awq_set_wait_timeout_ms(uint32_t ms) { g_timeout_ms.store(ms == 0 ? 1 : ms); }

void awq_profile_next_search(void *ev_begin, void *ev_end) {
    t_prof_begin = static_cast<cudaEvent_t>(ev_begin);
    t_prof_end = static_cast<cudaEvent_t>(ev_end);
}

awq_status awq_act_stats(const void *X, int64_t T, int64_t K, int64_t ldx, float *a, void *stream) {
    if (!X || !a || !aligned16(X) || !aligned16(a)) return AWQ_ERR_INVALID_ARG;
    if (T < 1 || T > kMaxDim || K < 8 || K > kMaxDim || K % 8 || ldx < K || ldx % 8) return AWQ_ERR_INVALID_ARG;
    DevInfo d;
    if (awq_status e = device_info(d)) return e;
    const int slabs = (int)((K + awq::kStatsCols - 1) / awq::kStatsCols);
    awq::act_stats_kernel<<<slabs * awq::kStatsCluster, awq::kStatsThreads, 0, (cudaStream_t)stream>>>(
        (const __half *)X, T, K, ldx, a);
    return last_launch();
}

awq_status awq_alpha_scales(const float *a, int64_t K, const float *alphas, int32_t n_alpha, float *s,
                            void *stream) {
    if (!a || !alphas || !s || !aligned16(a) || !aligned16(s) || !aligned16(alphas)) return AWQ_ERR_INVALID_ARG;
    if (K < 1 || K > kMaxDim || n_alpha < 1 || n_alpha > kMaxAlpha) return AWQ_ERR_INVALID_ARG;
    DevInfo d;
    if (awq_status e = device_info(d)) return e;
    const int grid = blocks_for((int64_t)n_alpha * K, 256);
    awq::alpha_scales_kernel<<<grid < 4 * d.sms ? grid : 4 * d.sms, 256, 0, (cudaStream_t)stream>>>(
        a, K, alphas, n_alpha, s, nullptr);
    return last_launch();
}

awq_status awq_quant_dequant(const void *W, int64_t N, int64_t K, const float *s, awq_qcfg q, void *W_hat,
                             void *stream) {
    return awq_quant_dequant_masked(W, N, K, s, q, nullptr, W_hat, stream);
}

awq_status awq_quant_dequant_masked(const void *W, int64_t N, int64_t K, const float *s, awq_qcfg q,
                                    const uint8_t *mask, void *W_hat, void *stream) {
    if (!W || !s || !W_hat || !aligned16(W) || !aligned16(s) || !aligned16(W_hat)) return AWQ_ERR_INVALID_ARG;
    if (!valid_qcfg(q) || N < 1 || N > kMaxDim || K < q.group_size || K > kMaxDim || K % q.group_size)
        return AWQ_ERR_INVALID_ARG;
    DevInfo d;
    if (awq_status e = device_info(d)) return e;
    const int G = (int)(K / q.group_size);
    const int tpg = q.group_size / 16;
    const int grid = blocks_for(N * G * tpg, 256);
    const float qmax = (float)((1 << q.bits) - 1);
    const int sym = q.zero_point ? 0 : 1;
    if (tpg == 8)
        awq::quant_dequant_kernel<8><<<grid, 256, 0, (cudaStream_t)stream>>>((const __half *)W, N, K, G, s, qmax, sym,
                                                                            mask, (__half *)W_hat);
    else
        awq::quant_dequant_kernel<4><<<grid, 256, 0, (cudaStream_t)stream>>>((const __half *)W, N, K, G, s, qmax, sym,
                                                                            mask, (__half *)W_hat);
    return last_launch();
}

size_t awq_search_workspace_bytes(int64_t N, int64_t K, int64_t T, awq_qcfg q, int32_t n_alpha) {
    if (!valid_qcfg(q) || N < 1 || K < 1 || T < 1 || n_alpha < 1 || K % q.group_size) return 0;
    return search_ws_layout(N, K, T, q.group_size, n_alpha).total;
}

awq_status awq_search_layer(const void *W, int64_t N, int64_t K, const void *X, int64_t T, int64_t ldx,
                            const float *a, awq_qcfg q, const float *alphas, int32_t n_alpha, float *losses,
                            float *row_losses, void *ws, size_t ws_bytes, void *stream) {
    return awq_search_layer_part(W, N, N, K, X, T, ldx, a, q, alphas, n_alpha, losses, row_losses, ws, ws_bytes,
                                 stream);
}

awq_status awq_search_layer_part(const void *W, int64_t N, int64_t rows_total, int64_t K, const void *X, int64_t T,
                                 int64_t ldx, const float *a, awq_qcfg q, const float *alphas, int32_t n_alpha,
                                 float *losses, float *row_losses, void *ws, size_t ws_bytes, void *stream) {
    if (!W || !X || !a || !alphas || !losses) return AWQ_ERR_INVALID_ARG;
    if (rows_total < N || rows_total > kMaxDim) return AWQ_ERR_INVALID_ARG;
    if (!aligned16(W) || !aligned16(X) || !aligned16(a) || !aligned16(alphas) || !aligned16(losses) ||
        (row_losses && !aligned16(row_losses)))
        return AWQ_ERR_INVALID_ARG;
    if (!valid_qcfg(q) || N < 1 || N > kMaxDim || T < 1 || T > kMaxDim || K < 64 || K > kMaxDim || K % 64 ||
        K % q.group_size || ldx < K || ldx % 8 || n_alpha < 1 || n_alpha > kMaxAlpha)
        return AWQ_ERR_INVALID_ARG;
    const SearchWs L = search_ws_layout(N, K, T, q.group_size, n_alpha);
    if (!ws || ws_bytes < L.total || (reinterpret_cast<uintptr_t>(ws) & 255u)) return AWQ_ERR_WORKSPACE;
    DevInfo d;
    if (awq_status e = device_info(d)) return e;
    cudaStream_t st = (cudaStream_t)stream;
    uint8_t *base = static_cast<uint8_t *>(ws);
    float *s_tab = reinterpret_cast<float *>(base + L.s_off);
    float *rs_tab = reinterpret_cast<float *>(base + L.rs_off);
    uint2 *params = reinterpret_cast<uint2 *>(base + L.prm_off);
    float *partial = reinterpret_cast<float *>(base + L.part_off);

    // a2: s and 1/s for every alpha
    {
        const int grid = blocks_for((int64_t)n_alpha * K, 256);
        awq::alpha_scales_kernel<<<grid < 4 * d.sms ? grid : 4 * d.sms, 256, 0, st>>>(a, K, alphas, n_alpha,
                                                                                     s_tab, rs_tab);
        if (awq_status e = last_launch()) return e;
    }
    return search_core(W, N, K, X, T, ldx, q, s_tab, rs_tab, n_alpha, nullptr, params, partial, losses, row_losses,
                       rows_total, d, st);
}


awq_status awq_search_layer_noalloc(const void *W, int64_t N, int64_t K, const void *X, int64_t T, int64_t ldx,
                                    const float *a, awq_qcfg q, const float *alphas, int32_t n_alpha,
                                    float *losses, float *row_losses, void *stream) {
    const size_t need = awq_search_workspace_bytes(N, K, T, q, n_alpha);
    if (need == 0) return AWQ_ERR_INVALID_ARG;
    if (need > AWQ_NOALLOC_SCRATCH_BYTES) return AWQ_ERR_WORKSPACE;
    DevInfo d;
    if (awq_status e = device_info(d)) return e;
    void *ws = nullptr;
    if (awq_status e = noalloc_scratch(&ws)) return e;
    return awq_search_layer(W, N, K, X, T, ldx, a, q, alphas, n_alpha, losses, row_losses, ws,
                            AWQ_NOALLOC_SCRATCH_BYTES, stream);
}

size_t awq_search_scales_workspace_bytes(int64_t N, int64_t K, int64_t T, awq_qcfg q, int32_t n_s, int32_t masked) {
    if (!valid_qcfg(q) || N < 1 || K < 1 || T < 1 || n_s < 1 || K % q.group_size) return 0;
    return search_ws_layout(N, K, T, q.group_size, n_s, masked != 0).total;
}

awq_status awq_search_scales(const void *W, int64_t N, int64_t K, const void *X, int64_t T, int64_t ldx,
                             awq_qcfg q, const float *s_table, int32_t n_s, const uint8_t *mask, float *losses,
                             float *row_losses, void *ws, size_t ws_bytes, void *stream) {
    if (!W || !X || !s_table || !losses) return AWQ_ERR_INVALID_ARG;
    if (!aligned16(W) || !aligned16(X) || !aligned16(s_table) || !aligned16(losses) ||
        (row_losses && !aligned16(row_losses)) || (mask && !aligned16(mask)))
        return AWQ_ERR_INVALID_ARG;
    if (!valid_qcfg(q) || N < 1 || N > kMaxDim || T < 1 || T > kMaxDim || K < 64 || K > kMaxDim || K % 64 ||
        K % q.group_size || ldx < K || ldx % 8 || n_s < 1 || n_s > kMaxAlpha)
        return AWQ_ERR_INVALID_ARG;
    const SearchWs L = search_ws_layout(N, K, T, q.group_size, n_s, mask != nullptr);
    if (!ws || ws_bytes < L.total || (reinterpret_cast<uintptr_t>(ws) & 255u)) return AWQ_ERR_WORKSPACE;
    DevInfo d;
    if (awq_status e = device_info(d)) return e;
    cudaStream_t st = (cudaStream_t)stream;
    uint8_t *base = static_cast<uint8_t *>(ws);
    float *s_tab = reinterpret_cast<float *>(base + L.s_off);
    float *rs_tab = reinterpret_cast<float *>(base + L.rs_off);
    uint2 *params = reinterpret_cast<uint2 *>(base + L.prm_off);
    float *partial = reinterpret_cast<float *>(base + L.part_off);
    {
        int grid = blocks_for((int64_t)n_s * K, 256);
        if (grid > 4 * d.sms) grid = 4 * d.sms;
        awq::scale_table_kernel<<<grid, 256, 0, st>>>(s_table, (int64_t)n_s * K, s_tab, rs_tab);
        if (awq_status e = last_launch()) return e;
    }
    const void *Xs = X;
    int64_t ld = ldx;
    if (mask) {                        // the fp16-kept channels take no part in the loss
        __half *Xm = reinterpret_cast<__half *>(base + L.xm_off);
        int grid = blocks_for(T * (K / 8), 256);
        if (grid > 8 * d.sms) grid = 8 * d.sms;
        awq::mask_columns_kernel<<<grid, 256, 0, st>>>((const __half *)X, T, K, ldx, mask, Xm);
        if (awq_status e = last_launch()) return e;
        Xs = Xm;
        ld = K;
    }
    return search_core(W, N, K, Xs, T, ld, q, s_tab, rs_tab, n_s, mask, params, partial, losses, row_losses, N, d,
                       st);
}

awq_status awq_salient_scales(const uint8_t *mask, int64_t K, float factor, float *s, void *stream) {
    if (!mask || !s || K < 1 || K > kMaxDim || !(factor > 0.0f && factor <= FLT_MAX)) return AWQ_ERR_INVALID_ARG;
    DevInfo d;
    if (awq_status e = device_info(d)) return e;
    int grid = blocks_for(K, 256);
    if (grid > 2 * d.sms) grid = 2 * d.sms;
    awq::salient_scales_kernel<<<grid, 256, 0, (cudaStream_t)stream>>>(mask, K, factor, s);
    return last_launch();
}

size_t awq_output_error_workspace_bytes(int64_t N, int64_t K, int64_t T) {
    if (N < 1 || K < 64 || T < 1 || K % 64) return 0;
    return search_ws_layout(N, K, T, 64, 1).total + round_up(2 * (size_t)N * K, 256);
}

awq_status awq_output_error(const void *W, const void *W_hat, int64_t N, int64_t K, const void *X, int64_t T,
                            int64_t ldx, float *loss, float *row_losses, void *ws, size_t ws_bytes, void *stream) {
    if (!W || !W_hat || !X || !loss) return AWQ_ERR_INVALID_ARG;
    if (!aligned16(W) || !aligned16(W_hat) || !aligned16(X) || !aligned16(loss) ||
        (row_losses && !aligned16(row_losses)))
        return AWQ_ERR_INVALID_ARG;
    if (N < 1 || N > kMaxDim || T < 1 || T > kMaxDim || K < 64 || K > kMaxDim || K % 64 || ldx < K || ldx % 8)
        return AWQ_ERR_INVALID_ARG;
    if (!ws || ws_bytes < awq_output_error_workspace_bytes(N, K, T) || (reinterpret_cast<uintptr_t>(ws) & 255u))
        return AWQ_ERR_WORKSPACE;
    DevInfo d;
    if (awq_status e = device_info(d)) return e;
    cudaStream_t st = (cudaStream_t)stream;
    const SearchWs L = search_ws_layout(N, K, T, 64, 1);
    uint8_t *base = static_cast<uint8_t *>(ws);
    float *s_tab = reinterpret_cast<float *>(base + L.s_off);
    float *rs_tab = reinterpret_cast<float *>(base + L.rs_off);
    uint2 *params = reinterpret_cast<uint2 *>(base + L.prm_off);
    float *partial = reinterpret_cast<float *>(base + L.part_off);
    __half *dW = reinterpret_cast<__half *>(base + L.total);
    int grid = blocks_for(N * K, 256);
    if (grid > 8 * d.sms) grid = 8 * d.sms;
    awq::weight_diff_kernel<<<grid, 256, 0, st>>>((const __half *)W, (const __half *)W_hat, N * K, dW);
    if (awq_status e = last_launch()) return e;
    const int64_t n_prm = (K / 64) * padded_rows(N);
    awq::zero_code_params_kernel<<<blocks_for(n_prm, 256) < 4 * d.sms ? blocks_for(n_prm, 256) : 4 * d.sms, 256, 0,
                                   st>>>(params, n_prm);
    if (awq_status e = last_launch()) return e;
    awq::fill_kernel<<<blocks_for(K, 256), 256, 0, st>>>(s_tab, K, 1.0f);
    awq::fill_kernel<<<blocks_for(K, 256), 256, 0, st>>>(rs_tab, K, 1.0f);
    if (awq_status e = last_launch()) return e;
    return run_search(dW, N, K, X, T, ldx, 64, 0.0f, s_tab, rs_tab, 1, params, partial, loss, row_losses, N, d, st);
}

awq_status awq_gptq_hessian(const void *X, int64_t T, int64_t K, int64_t ldx, const float *s, float *H, void *stream) {
    if (!X || !s || !H || !aligned16(X) || !aligned16(s) || !aligned16(H)) return AWQ_ERR_INVALID_ARG;
    if (T < 1 || T > kMaxDim || K < 64 || K > kMaxGptqK || K % 64 || ldx < K || ldx % 8) return AWQ_ERR_INVALID_ARG;
    DevInfo d;
    if (awq_status e = device_info(d)) return e;
    const int nb = (int)(K / awq::kGb);
    awq::gptq_hessian_kernel<<<nb * (nb + 1) / 2, 256, 0, (cudaStream_t)stream>>>((const __half *)X, T, K, ldx, s, H);
    return last_launch();
}

size_t awq_gptq_hessian_workspace_bytes(int64_t T, int64_t K) {
    if (T < 1 || T > kMaxDim || K < 64 || K % 64 || K > kMaxGptqK) return 0;
    const int64_t Tp = (T + awq::ghs::TS - 1) / awq::ghs::TS * awq::ghs::TS;
    return round_up(2 * 3 * (size_t)K * (size_t)Tp, 256);
}

awq_status awq_gptq_hessian_tc(const void *X, int64_t T, int64_t K, int64_t ldx, const float *s, float *H, void *ws,
                               size_t ws_bytes, void *stream) {
    if (!X || !s || !H || !aligned16(X) || !aligned16(s) || !aligned16(H)) return AWQ_ERR_INVALID_ARG;
    if (T < 1 || T > kMaxDim || K < 64 || K > kMaxGptqK || K % 64 || ldx < K || ldx % 8) return AWQ_ERR_INVALID_ARG;
    if (!ws || ws_bytes < awq_gptq_hessian_workspace_bytes(T, K) || (reinterpret_cast<uintptr_t>(ws) & 255u))
        return AWQ_ERR_WORKSPACE;
    DevInfo d;
    if (awq_status e = device_info(d)) return e;
    cudaStream_t st = (cudaStream_t)stream;
    const int64_t Tp = (T + awq::ghs::TS - 1) / awq::ghs::TS * awq::ghs::TS;
    __nv_bfloat16 *xt = static_cast<__nv_bfloat16 *>(ws);
    const dim3 pgrid((unsigned)((K + awq::ghs::XT_TILE - 1) / awq::ghs::XT_TILE),
                     (unsigned)((Tp + awq::ghs::XT_TILE - 1) / awq::ghs::XT_TILE));
    awq::gptq_hprep_kernel<<<pgrid, 256, 0, st>>>((const __half *)X, T, K, ldx, Tp, s, xt);
    if (awq_status e = last_launch()) return e;
    CUtensorMap tmap;
    if (!encode_bf16_map(&tmap, xt, 3 * K, Tp, awq::ghs::TB)) return AWQ_ERR_CUDA;
    const int nb = (int)((K + awq::ghs::TB - 1) / awq::ghs::TB);
    const int n_tiles = nb * (nb + 1) / 2;
    const int grid = n_tiles < d.sms ? n_tiles : d.sms;
    awq::gptq_hessian_tc_kernel<<<grid, awq::ghs::THREADS, awq::ghs::SMEM_BYTES, st>>>(
        tmap, K, Tp / awq::ghs::TS, H, (uint64_t)g_timeout_ms.load() * 1000000ull);
    return last_launch();
}

size_t awq_gptq_factor_workspace_bytes(int64_t K) {
    if (K < 64 || K % 64 || K > kMaxGptqK) return 0;
    return round_up(4 * (size_t)K * K, 256) + 256;
}

awq_status awq_gptq_factor(const float *H, int64_t K, float damp, float *U, void *ws, size_t ws_bytes, void *stream) {
    if (!H || !U || !aligned16(H) || !aligned16(U)) return AWQ_ERR_INVALID_ARG;
    if (K < 64 || K % 64 || K > kMaxGptqK || !(damp >= 0.0f && damp <= 1e6f)) return AWQ_ERR_INVALID_ARG;
    if (!ws || ws_bytes < awq_gptq_factor_workspace_bytes(K) || (reinterpret_cast<uintptr_t>(ws) & 255u))
        return AWQ_ERR_WORKSPACE;
    DevInfo d;
    if (awq_status e = device_info(d)) return e;
    cudaStream_t st = (cudaStream_t)stream;
    float *A = static_cast<float *>(ws);
    float *add = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + round_up(4 * (size_t)K * K, 256));
    awq::gptq_damp_kernel<<<1, 256, 0, st>>>(H, K, damp, add);
    int grid = blocks_for(K * K, 256);
    if (grid > 8 * d.sms) grid = 8 * d.sms;
    awq::gptq_reverse_kernel<<<grid, 256, 0, st>>>(H, K, add, A);
    if (awq_status e = last_launch()) return e;
    const int nb = (int)(K / awq::kGb);
    for (int p = 0; p < nb; ++p) {          // blocked Cholesky of the reversed, damped Hessian
        awq::chol_diag_kernel<<<1, awq::kCholDiagThreads, 0, st>>>(A, K, p);
        const int m = nb - p - 1;
        if (m > 0) {
            awq::chol_panel_kernel<<<m, awq::kGb, 0, st>>>(A, K, p);
            awq::chol_update_kernel<<<m * (m + 1) / 2, 256, 0, st>>>(A, K, p);
        }
        if (awq_status e = last_launch()) return e;
    }
    // M = L^-1 into U's storage: diagonal blocks, then block rows in order,
    // the pending sums of the rows below kept in the blocks they will become
    if (cudaMemsetAsync(U, 0, 4 * (size_t)K * K, st) != cudaSuccess) return AWQ_ERR_CUDA;
    awq::trinv_diag_kernel<<<nb, awq::kGb, 0, st>>>(A, K, U);
    for (int k = 0; k < nb; ++k) {
        if (k > 0) awq::trinv_final_kernel<<<k, 256, 0, st>>>(K, k, U);
        if (k + 1 < nb) awq::trinv_update_kernel<<<(nb - 1 - k) * (k + 1), 256, 0, st>>>(A, K, k, U);
        if (awq_status e = last_launch()) return e;
    }
    grid = blocks_for((K * K + 1) / 2, 256);
    if (grid > 8 * d.sms) grid = 8 * d.sms;
    awq::gptq_rotate_kernel<<<grid, 256, 0, st>>>(U, K);                 // U = P M P, upper part
    return last_launch();
}

awq_status awq_gptq_quantize(const void *W, int64_t N, int64_t K, const float *s, const float *U, awq_qcfg q,
                             uint32_t *codes, void *scales, void *zeros, void *W_hat, void *stream) {
    if (!W || !s || !U || !codes || !scales || !zeros || !W_hat) return AWQ_ERR_INVALID_ARG;
    if (!aligned16(W) || !aligned16(s) || !aligned16(U) || !aligned16(codes) || !aligned16(scales) ||
        !aligned16(zeros) || !aligned16(W_hat))
        return AWQ_ERR_INVALID_ARG;
    if (!valid_qcfg(q) || N < 1 || N > kMaxDim || K < 64 || K % 64 || K > kMaxGptqK || K % q.group_size)
        return AWQ_ERR_INVALID_ARG;
    DevInfo d;
    if (awq_status e = device_info(d)) return e;
    awq::gsw::Args A;
    A.W = (const __half *)W;
    A.N = N;
    A.K = K;
    A.s = s;
    A.U = U;
    A.group = q.group_size;
    A.G = (int)(K / q.group_size);
    A.bits = q.bits;
    A.sym = q.zero_point ? 0 : 1;
    A.qmax = (float)((1 << q.bits) - 1);
    A.codes = codes;
    A.scales = (__half *)scales;
    A.zeros = (__half *)zeros;
    A.W_hat = (__half *)W_hat;
    A.timeout_ns = (uint64_t)g_timeout_ms.load() * 1000000ull;
    // the block's 256 worker threads own column pairs of R rows in registers:
    // pairs per thread and rows per block trade against each other, and past
    // K = 4096 two-column batches keep the ring of U rows in shared memory
    const int bw = K <= 4096 ? 4 : 2;
    const int rows = K <= 4096 ? 8 : 4;
    A.ring = 2;                                  // deeper rings measured no faster: the batch's serial part bounds it
    const size_t smem = awq::gsw::smem_bytes(K, rows, bw, A.ring);
    if (smem > (size_t)awq::qlv::SMEM_LIMIT) return AWQ_ERR_UNSUPPORTED;
    cudaStream_t st = (cudaStream_t)stream;
#define AWQ_SWEEP(SLOTS, R, B)                                                                            \
    awq::gptq_sweep_kernel<SLOTS, R, B><<<(unsigned)((N + R - 1) / R), awq::gsw::THREADS, smem, st>>>(A)
    if (K <= 512) AWQ_SWEEP(1, 8, 4);
    else if (K <= 1024) AWQ_SWEEP(2, 8, 4);
    else if (K <= 2048) AWQ_SWEEP(4, 8, 4);
    else if (K <= 4096) AWQ_SWEEP(8, 8, 4);
    else AWQ_SWEEP(16, 4, 2);
#undef AWQ_SWEEP
    return last_launch();
}

awq_status awq_channel_topk(const float *stat, int64_t K, int64_t k, uint8_t *mask, void *stream) {
    if (!stat || !mask || K < 1 || K > kMaxDim || k < 0 || k > K) return AWQ_ERR_INVALID_ARG;
    DevInfo d;
    if (awq_status e = device_info(d)) return e;
    const int grid = blocks_for(K, awq::kTopkThreads);
    awq::topk_kernel<<<grid, awq::kTopkThreads, 0, (cudaStream_t)stream>>>(stat, K, k, mask);
    return last_launch();
}

awq_status awq_pack(const void *W, int64_t N, int64_t K, const float *a, awq_qcfg q, const float *alphas,
                    const float *losses, int32_t n_alpha, int32_t *best_idx, float *s_best, uint32_t *codes,
                    void *scales, void *zeros, void *stream) {
    if (!W || !a || !alphas || !losses || !best_idx || !s_best || !codes || !scales || !zeros)
        return AWQ_ERR_INVALID_ARG;
    if (!aligned16(W) || !aligned16(a) || !aligned16(s_best) || !aligned16(codes) || !aligned16(scales) ||
        !aligned16(zeros) || !aligned16(alphas) || !aligned16(losses) || !aligned16(best_idx))
        return AWQ_ERR_INVALID_ARG;
    if (!valid_qcfg(q) || N < 1 || N > kMaxDim || K < q.group_size || K > kMaxDim || K % q.group_size ||
        n_alpha < 1 || n_alpha > kMaxAlpha)
        return AWQ_ERR_INVALID_ARG;
    DevInfo d;
    if (awq_status e = device_info(d)) return e;
    cudaStream_t st = (cudaStream_t)stream;
    {
        int grid = blocks_for(K, 256);
        if (grid > 2 * d.sms) grid = 2 * d.sms;
        awq::best_scale_kernel<<<grid, 256, 0, st>>>(a, K, alphas, losses, n_alpha, best_idx, s_best);
        if (awq_status e = last_launch()) return e;
    }
    return launch_pack(W, N, K, s_best, q, codes, scales, zeros, st);
}

awq_status awq_pack_scales(const void *W, int64_t N, int64_t K, const float *s, awq_qcfg q, uint32_t *codes,
                           void *scales, void *zeros, void *stream) {
    if (!W || !s || !codes || !scales || !zeros) return AWQ_ERR_INVALID_ARG;
    if (!aligned16(W) || !aligned16(s) || !aligned16(codes) || !aligned16(scales) || !aligned16(zeros))
        return AWQ_ERR_INVALID_ARG;
    if (!valid_qcfg(q) || N < 1 || N > kMaxDim || K < q.group_size || K > kMaxDim || K % q.group_size)
        return AWQ_ERR_INVALID_ARG;
    DevInfo d;
    if (awq_status e = device_info(d)) return e;
    return launch_pack(W, N, K, s, q, codes, scales, zeros, (cudaStream_t)stream);
}

size_t awq_qlinear_workspace_bytes(int64_t T, int64_t K, int64_t N) {
    if (T < 1 || K < 1 || N < 1) return 0;
    return qlinear_ws(T, K, N);
}

awq_status awq_qlinear_cc(const uint32_t *codes, const void *scales, const void *zeros, const float *s_best,
                          int64_t N, int64_t K, awq_qcfg q, const void *X, int64_t T, int64_t ldx, float *Y,
                          void *ws, size_t ws_bytes, void *stream) {
    if (!codes || !scales || !zeros || !s_best || !X || !Y) return AWQ_ERR_INVALID_ARG;
    if (!aligned16(codes) || !aligned16(scales) || !aligned16(zeros) || !aligned16(s_best) || !aligned16(X) ||
        !aligned16(Y))
        return AWQ_ERR_INVALID_ARG;
    if (!valid_qcfg(q) || N < 1 || N > kMaxDim || T < 1 || T > kMaxDim || K < 64 || K > kMaxDim || K % 64 ||
        K % q.group_size || ldx < K || ldx % 8)
        return AWQ_ERR_INVALID_ARG;
    if (!ws || ws_bytes < qlinear_ws(T, K, N) || (reinterpret_cast<uintptr_t>(ws) & 255u)) return AWQ_ERR_WORKSPACE;
    DevInfo d;
    if (awq_status e = device_info(d)) return e;
    cudaStream_t st = (cudaStream_t)stream;
    const bool c2 = q.bits == 2;
    const int64_t cpw = c2 ? 16 : 8;                       // codes per 32-bit word
    const int64_t sc = awq::qlv::WORDS * cpw;              // columns per stage
    const int64_t Kp = ql_cols_pad(K, sc), T_pad = ql_rows_pad(T);
    const int64_t row_blocks = ql_row_blocks(N);
    uint8_t *w8 = static_cast<uint8_t *>(ws);
    float *xs = reinterpret_cast<float *>(w8);
    float *part = reinterpret_cast<float *>(w8 + ql_xs_bytes(T, K));
    unsigned *cnt = reinterpret_cast<unsigned *>(w8 + ql_xs_bytes(T, K) + ql_part_bytes(N));
    {
        int grid = blocks_for(T_pad * Kp / 4, 256);
        if (grid > 4 * d.sms) grid = 4 * d.sms;
        awq::qlinear_prep_kernel<<<grid, 256, 0, st>>>((const __half *)X, T, T_pad, K, Kp, ldx, (int)cpw, s_best,
                                                       xs, cnt, row_blocks * awq::qlv::RGROUPS);
        if (awq_status e = last_launch()) return e;
    }
    CUtensorMap tmap;
    if (!encode_codes_map(&tmap, codes, N, K / cpw)) return AWQ_ERR_CUDA;
    awq::qlv::Args A;
    A.Kp = Kp;
    A.scales = (const __half *)scales;
    A.zeros = (const __half *)zeros;
    A.N = N;
    A.K = K;
    A.G = (int)(K / q.group_size);
    A.group = q.group_size;
    A.n_steps = Kp / sc;
    A.units = row_blocks * A.n_steps;
    A.gps = (int)(sc / q.group_size);
    A.sz_mode = A.G % 8 == 0 ? 16 : (A.G % 2 == 0 ? 4 : 2);
    // tokens per pass: 1, 2, or 4 (every pass reads the codes once; a last pass
    // with fewer tokens reads the zero rows that pad x')
    const int tt = T == 1 ? 1 : (T == 2 || c2) ? 2 : awq::qlv::TOKENS;   // 2-bit words: at most 2 tokens
    A.n_stages = awq::qlv::ring_stages((int)sc, tt, A.gps);
    const size_t smem = (size_t)A.n_stages * awq::qlv::stage_bytes((int)sc, tt, A.gps) + awq::qlv::fixed_smem();
    A.part = part;
    A.cnt = cnt;
    A.timeout_ns = (uint64_t)g_timeout_ms.load() * 1000000ull;
    // one block per SM, each streaming an equal share of the units
    int64_t grid = d.sms < kQlMaxGrid ? d.sms : kQlMaxGrid;
    if (grid > A.units) grid = A.units;
    for (int64_t t0 = 0; t0 < T; t0 += tt) {
        A.xs = xs + t0 * Kp;
        A.Y = Y + t0 * N;
        A.T = (int)(T - t0 < tt ? T - t0 : tt);
#define AWQ_QL_LAUNCH(CB, TT) \
    awq::qlinear_gemv_kernel<CB, TT><<<(unsigned)grid, awq::qlv::THREADS, smem, st>>>(tmap, A)
        if (tt == 1) { if (c2) AWQ_QL_LAUNCH(2, 1); else AWQ_QL_LAUNCH(4, 1); }
        else if (tt == 2) { if (c2) AWQ_QL_LAUNCH(2, 2); else AWQ_QL_LAUNCH(4, 2); }
        else AWQ_QL_LAUNCH(4, 4);
#undef AWQ_QL_LAUNCH
        if (awq_status e = last_launch()) return e;
    }
    return AWQ_OK;
}

awq_status awq_qlinear_tc(const uint32_t *codes, const void *scales, const void *zeros, const float *s_best,
                          int64_t N, int64_t K, awq_qcfg q, const void *X, int64_t T, int64_t ldx, float *Y,
                          void *ws, size_t ws_bytes, void *stream) {
    if (!codes || !scales || !zeros || !s_best || !X || !Y) return AWQ_ERR_INVALID_ARG;
    if (!aligned16(codes) || !aligned16(scales) || !aligned16(zeros) || !aligned16(s_best) || !aligned16(X) ||
        !aligned16(Y))
        return AWQ_ERR_INVALID_ARG;
    if (!valid_qcfg(q) || N < 1 || N > kMaxDim || T < 1 || T > kMaxDim || K < 64 || K > kMaxDim || K % 64 ||
        K % q.group_size || ldx < K || ldx % 8)
        return AWQ_ERR_INVALID_ARG;
    if (!ws || ws_bytes < qlinear_ws(T, K, N) || (reinterpret_cast<uintptr_t>(ws) & 255u)) return AWQ_ERR_WORKSPACE;
    DevInfo d;
    if (awq_status e = device_info(d)) return e;
    cudaStream_t st = (cudaStream_t)stream;
    const QtcPlan P = qtc_plan(T, K, N, q.group_size);
    const int G = (int)(K / q.group_size);
    uint8_t *w8 = static_cast<uint8_t *>(ws);
    __nv_bfloat16 *xb = reinterpret_cast<__nv_bfloat16 *>(w8);
    float *gsum = reinterpret_cast<float *>(w8 + P.xb_bytes);
    float *part = reinterpret_cast<float *>(w8 + P.xb_bytes + P.gs_bytes);
    unsigned *cnt = reinterpret_cast<unsigned *>(w8 + P.xb_bytes + P.gs_bytes + P.part_bytes);
    {
        const int64_t work = std::max((int64_t)P.n_pass * P.NR * P.Kp, (int64_t)P.n_pass * G * 16 * 16);
        int grid = blocks_for(work, 256);
        if (grid > 8 * d.sms) grid = 8 * d.sms;
        awq::qtc_prep_kernel<<<grid, 256, 0, st>>>((const __half *)X, T, K, P.Kp, ldx, s_best, P.TT, P.NR, P.n_pass,
                                                   G, q.group_size, xb, gsum, cnt, P.row_blocks * 4);
        if (awq_status e = last_launch()) return e;
    }
    const bool c2 = q.bits == 2;
    const int cpw = c2 ? 16 : 8;
    CUtensorMap tmap_codes, tmap_b;
    if (!encode_words_map(&tmap_codes, codes, N, K / cpw, c2 ? 16 : 32, awq::qtc::ROWS) ||
        !encode_bf16_map(&tmap_b, xb, (int64_t)P.n_pass * P.NR, P.Kp, P.NR))
        return AWQ_ERR_CUDA;
    awq::qtc::Args A;
    A.scales = (const __half *)scales;
    A.zeros = (const __half *)zeros;
    A.N = N;
    A.G = G;
    A.n_steps = P.n_steps;
    A.units = P.units;
    A.part = part;
    A.cnt = cnt;
    A.timeout_ns = (uint64_t)g_timeout_ms.load() * 1000000ull;
    int64_t grid = d.sms < kQlMaxGrid ? d.sms : kQlMaxGrid;
    if (grid > P.units) grid = P.units;
    const bool g64 = q.group_size == 64;
    for (int pass = 0; pass < P.n_pass; ++pass) {
        A.gsum = gsum + (int64_t)pass * G * 16;
        A.Y = Y + (int64_t)pass * P.TT * N;
        A.T = (int)(T - (int64_t)pass * P.TT < P.TT ? T - (int64_t)pass * P.TT : P.TT);
        A.b_row0 = pass * P.NR;
        const unsigned g = (unsigned)grid;
        cudaError_t err;
#define AWQ_QTC_LAUNCH(NR, CB, GPS) err = launch_qtc<NR, CB, GPS>(g, st, tmap_codes, tmap_b, A)
#define AWQ_QTC_BY_CODE(NR)                                                   \
    do {                                                                      \
        if (c2) { if (g64) AWQ_QTC_LAUNCH(NR, 2, 4); else AWQ_QTC_LAUNCH(NR, 2, 2); } \
        else { if (g64) AWQ_QTC_LAUNCH(NR, 4, 4); else AWQ_QTC_LAUNCH(NR, 4, 2); }    \
    } while (0)
        if (P.NR == 16) AWQ_QTC_BY_CODE(16);
        else if (P.NR == 32) AWQ_QTC_BY_CODE(32);
        else AWQ_QTC_BY_CODE(48);
#undef AWQ_QTC_BY_CODE
#undef AWQ_QTC_LAUNCH
        if (err != cudaSuccess) return AWQ_ERR_CUDA;
        if (awq_status e = last_launch()) return e;
    }
    return AWQ_OK;
}

// From kQlTcMinTokens tokens on, one tensor-core pass reads the codes once for
// up to 16 tokens, where the CUDA-core kernel reads them once per 1, 2 or 4.
int32_t awq_qlinear_path(int64_t T) { return T >= kQlTcMinTokens ? 1 : 0; }

awq_status awq_qlinear(const uint32_t *codes, const void *scales, const void *zeros, const float *s_best,
                       int64_t N, int64_t K, awq_qcfg q, const void *X, int64_t T, int64_t ldx, float *Y,
                       void *ws, size_t ws_bytes, void *stream) {
    if (awq_qlinear_path(T) == 1)
        return awq_qlinear_tc(codes, scales, zeros, s_best, N, K, q, X, T, ldx, Y, ws, ws_bytes, stream);
    return awq_qlinear_cc(codes, scales, zeros, s_best, N, K, q, X, T, ldx, Y, ws, ws_bytes, stream);
}

awq_status awq_selftest_bounded_wait(void *stream) {
    DevInfo d;
    if (awq_status e = device_info(d)) return e;
    awq::selftest_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>((uint64_t)g_timeout_ms.load() * 1000000ull);
    return last_launch();
}

awq_status awq_get_status(void *stream) {
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return AWQ_ERR_CUDA;
    unsigned flags = 0;
    if (cudaMemcpyFromSymbol(&flags, awq::g_dev_error, sizeof(flags)) != cudaSuccess) return AWQ_ERR_CUDA;
    if (flags) {
        const unsigned zero = 0;
        if (cudaMemcpyToSymbol(awq::g_dev_error, &zero, sizeof(zero)) != cudaSuccess) return AWQ_ERR_CUDA;
        if (flags & awq::kDevErrTimeout) return AWQ_ERR_TIMEOUT;
        if (flags & (awq::kDevErrBadAlpha | awq::kDevErrBadScale | awq::kDevErrNotPD)) return AWQ_ERR_INVALID_ARG;
    }
    return last_launch();
}

}  // extern "C"

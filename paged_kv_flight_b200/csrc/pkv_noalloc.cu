// pkv_noalloc.cu -- pkv_decode_attn_noalloc: the decode attention of
// pkv_decode_attn for callers that may not allocate device memory.
//
// Some callers cannot call cudaMalloc: a serving runtime that reserved all
// device memory for its own pool at start-up (a later cudaMalloc fails or
// breaks its accounting), a plug-in that may only use memory handed to it by
// its host framework, or a latency-critical path that must not pay for an
// allocation and the device synchronisation that can come with it.  Creating a
// context (pkv_create) allocates the attention workspace; this entry point
// allocates nothing.  Its scratch (split partials, the split geometry the
// attention kernel hands to the combine kernel, the device error word) lives
// in one file-scope device
// array of kScratchBytes that every GPU that loads this library holds until
// the process exits.
//
// Set-up, once per device, on the first call made while that device is
// current: the device address of the array is looked up with
// cudaGetSymbolAddress and cached, with the SM count and the attention
// kernel's attributes (set once per head_dim / KV type).  That first call
// should therefore come before any stream capture.  Every call shares the one array, which keeps
// the previous call's contents: the error word is cleared with
// cudaMemsetAsync on the caller's stream at each call, and everything else is
// written before it is read within the call, so calls ordered
// on one stream are independent, but calls that overlap on the GPU (different
// streams, or different host threads without ordering) race on the array.
// Device-side range errors (page id or length out of range) are handled as in
// pkv_decode_attn (the affected work is skipped) but cannot be read back:
// there is no context.
#include <math.h>
#include <mutex>

#include <cudaTypedefs.h>

#include "pkv_internal.h"

namespace {

constexpr size_t kScratchBytes = 16u << 20;      // 16 MiB per device
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_setup_mutex;

// Per-device state set up once, under g_setup_mutex, with the device current:
// the scratch array's device address, the SM count, and the attention launch
// shape (kernel attributes set then) of each (head_dim, KV type, tile) variant.
struct DeviceSetup {
    void* scratch = nullptr;
    int num_sms = 0;
    bool launch_ready[2][2][2] = {};          // [head_dim 128][E4M3][32-token tiles]
    pkv::AttnLaunch launch[2][2][2];
};
DeviceSetup g_setup[kMaxDevices];

// The current device's set-up, with the launch shape for cfg in *L; nullptr
// on failure.
const DeviceSetup* setup_current_device(const pkv_config* cfg, pkv::AttnLaunch* L)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    DeviceSetup& s = g_setup[dev];
    if (!s.scratch) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
            return nullptr;
        s.num_sms = sms;
        s.scratch = ptr;
    }
    const bool fp8 = cfg->kv_dtype == PKV_KV_FP8_E4M3;
    const int i = cfg->head_dim == 128, j = fp8 ? 1 : 0, k = pkv::attn_tile(fp8, cfg->page_size) == pkv::kTileWide;
    if (!s.launch_ready[i][j][k]) {
        // sized for the largest batch: the kernel's shared-memory limit is the
        // same one every context sets, so this never lowers it
        if (pkv::attn_prepare(cfg->head_dim, fp8, cfg->page_size, s.num_sms, pkv::kMaxBatch, &s.launch[i][j][k]) !=
            cudaSuccess)
            return nullptr;
        s.launch_ready[i][j][k] = true;
    }
    *L = s.launch[i][j][k];
    return &s;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

pkv_status check_config(const pkv_config* c)
{
    if (!c) return PKV_ERR_INVALID_ARG;
    if (c->num_q_heads <= 0 || c->num_kv_heads <= 0 || c->num_q_heads % c->num_kv_heads) return PKV_ERR_INVALID_ARG;
    if (c->head_dim <= 0 || c->page_size <= 0) return PKV_ERR_INVALID_ARG;
    if (c->kv_dtype != PKV_KV_BF16 && c->kv_dtype != PKV_KV_FP8_E4M3) return PKV_ERR_INVALID_ARG;
    if (c->max_batch <= 0 || c->max_blocks_per_seq <= 0 || c->num_pages <= 0) return PKV_ERR_INVALID_ARG;
    if ((long long)c->max_blocks_per_seq * c->page_size >= (1LL << 31)) return PKV_ERR_INVALID_ARG;
    if (c->num_q_heads / c->num_kv_heads > pkv::kMaxGroup) return PKV_ERR_UNSUPPORTED;
    if (c->head_dim != 64 && c->head_dim != 128) return PKV_ERR_UNSUPPORTED;
    if (c->page_size != 16 && c->page_size != 32 && c->page_size != 64) return PKV_ERR_UNSUPPORTED;
    if (c->max_batch > pkv::kMaxBatch) return PKV_ERR_UNSUPPORTED;
    if ((long long)c->num_pages * c->num_kv_heads * c->page_size >= (1LL << 31)) return PKV_ERR_UNSUPPORTED;
    return PKV_OK;
}

bool encode_pool(const pkv_config* c, const void* pool, CUtensorMap* map)
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return false;
        fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    const bool fp8 = c->kv_dtype == PKV_KV_FP8_E4M3;
    const int elem = fp8 ? 1 : 2;
    const int rowb = c->head_dim * elem;
    const int boxb = rowb > 128 ? 128 : rowb;
    cuuint64_t dims[2] = {(cuuint64_t)c->head_dim, (cuuint64_t)c->num_pages * c->num_kv_heads * c->page_size};
    cuuint64_t strides[1] = {(cuuint64_t)rowb};
    cuuint32_t box[2] = {(cuuint32_t)(boxb / elem), (cuuint32_t)pkv::attn_tile(fp8, c->page_size)};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
              const_cast<void*>(pool), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              boxb == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

extern "C" pkv_status pkv_decode_attn_noalloc(const pkv_config* cfg, const void* q, const void* k_pool,
                                              const void* v_pool, const float* k_scale, const float* v_scale,
                                              const int32_t* block_tables, int bt_stride,
                                              const int32_t* seq_lens, int batch, void* out,
                                              cudaStream_t stream)
{
    const pkv_status v = check_config(cfg);
    if (v != PKV_OK) return v;
    if (batch < 0 || batch > cfg->max_batch) return PKV_ERR_INVALID_ARG;
    if (batch == 0) return PKV_OK;
    if (bt_stride <= 0 || bt_stride > cfg->max_blocks_per_seq) return PKV_ERR_INVALID_ARG;
    if (!q || !out || !k_pool || !v_pool || !block_tables || !seq_lens) return PKV_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(out) || !aligned16(k_pool) || !aligned16(v_pool) || !aligned16(block_tables) ||
        !aligned16(seq_lens))
        return PKV_ERR_INVALID_ARG;
    const bool fp8 = cfg->kv_dtype == PKV_KV_FP8_E4M3;
    if (fp8 && (!k_scale || !v_scale || !aligned16(k_scale) || !aligned16(v_scale))) return PKV_ERR_INVALID_ARG;

    pkv::AttnLaunch L;
    const DeviceSetup* setup = setup_current_device(cfg, &L);
    if (!setup) return PKV_ERR_CUDA;

    // scratch layout: [error word, chunk counter | split geometry | partial rows | partial (m, l)];
    // a static split (no dynamic tail): two partial slots per warp
    const size_t workers = (size_t)setup->num_sms * pkv::kAttnWarps;
    const size_t b_err = 256;
    const size_t b_cnt = ((size_t)(batch + 8) * sizeof(int) + 255) & ~(size_t)255;
    const size_t b_po = 2 * workers * pkv::kMaxGroup * cfg->head_dim * sizeof(float);
    const size_t b_pml = 2 * workers * pkv::kMaxGroup * 2 * sizeof(float);
    if (b_err + b_cnt + b_po + b_pml > kScratchBytes) return PKV_ERR_UNSUPPORTED;   // beyond the fixed scratch
    unsigned char* base = static_cast<unsigned char*>(setup->scratch);

    CUtensorMap tmk, tmv;
    if (!encode_pool(cfg, k_pool, &tmk) || !encode_pool(cfg, v_pool, &tmv)) return PKV_ERR_CUDA;

    // the previous call may have left anything here: clear what must start at zero
    if (cudaMemsetAsync(base, 0, b_err, stream) != cudaSuccess) return PKV_ERR_CUDA;

    pkv::AttnParams p;
    p.q = static_cast<const __nv_bfloat16*>(q);
    p.out = static_cast<__nv_bfloat16*>(out);
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    p.block_tables = block_tables;
    p.seq_lens = seq_lens;
    p.err = reinterpret_cast<int*>(base);
    p.claim = reinterpret_cast<int*>(base + 128);
    p.meta = reinterpret_cast<int*>(base + b_err);
    p.part_o = reinterpret_cast<float*>(base + b_err + b_cnt);
    p.part_ml = reinterpret_cast<float*>(base + b_err + b_cnt + b_po);
    p.scale_log2 = (float)(1.4426950408889634 / sqrt((double)cfg->head_dim));
    p.batch = batch;
    p.bt_stride = bt_stride;
    p.Hq = cfg->num_q_heads;
    p.Hkv = cfg->num_kv_heads;
    p.G = cfg->num_q_heads / cfg->num_kv_heads;
    p.P = cfg->page_size;
    p.num_pages = cfg->num_pages;
    p.stages = L.stages;
    p.workers = 0;
    p.tail_chunks = 0;
    p.q_len = 1;
    return pkv::launch_decode_attn(p, tmk, tmv, cfg->head_dim, fp8, L, stream) == cudaSuccess ? PKV_OK
                                                                                              : PKV_ERR_CUDA;
}

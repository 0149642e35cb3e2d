// lca_api.cu -- the C ABI declared in include/lca.h: argument checks,
// workspace layout, TMA tensor maps and kernel launches.  All kernels are in
// this one translation unit (the .cuh files it includes).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <utility>
#include <vector>

#include "../../include/lca.h"
#include "common.cuh"
#include "prep_combine.cuh"
#include "condense.cuh"
#include "attn_decode.cuh"
#include "wuv_gemm.cuh"
#include "prefill.cuh"
#include "selftest.cuh"
#include "varlen.cuh"
#include "append.cuh"

using namespace lca;

namespace {

constexpr int kMaxCtas = 256;      // split-L grid cap; sizes the partial buffers
constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ------------------------------------------------------------------ device
struct DeviceInfo {
    int sms = 0;
    bool ok = false;
    bool attrs_set = false;
};
std::mutex g_mu;
DeviceInfo g_dev[64];

int current_device(DeviceInfo **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return LCA_ERR_NO_DEVICE;
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceInfo &d = g_dev[dev];
    if (!d.ok) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return LCA_ERR_NO_DEVICE;
        if (major != 10 || minor != 0) return LCA_ERR_NO_DEVICE;
        d.sms = sms;
        d.ok = true;
    }
    if (!d.attrs_set) {
        bool good = true;
        good &= cudaFuncSetAttribute(attn_decode_kernel<MODE_MLA>, cudaFuncAttributeMaxDynamicSharedMemorySize, AT_SMEM_ALLOC) == cudaSuccess;
        good &= cudaFuncSetAttribute(attn_decode_kernel<MODE_REPS>, cudaFuncAttributeMaxDynamicSharedMemorySize, AT_SMEM_ALLOC) == cudaSuccess;
        good &= cudaFuncSetAttribute(attn_decode_kernel<MODE_LCA>, cudaFuncAttributeMaxDynamicSharedMemorySize, AT_SMEM_ALLOC) == cudaSuccess;
        good &= cudaFuncSetAttribute(attn_decode_kernel<MODE_MLA, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, AT_SMEM_ALLOC) == cudaSuccess;
        good &= cudaFuncSetAttribute(attn_decode_kernel<MODE_LCA, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, AT_SMEM_ALLOC) == cudaSuccess;
        good &= cudaFuncSetAttribute(attn_decode_kernel<MODE_REPS, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, AT_SMEM_ALLOC) == cudaSuccess;
        good &= cudaFuncSetAttribute(condense_kernel<CdShape::kWarps, CdShape::kSlots>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, CdShape::kSmem) == cudaSuccess;
        good &= cudaFuncSetAttribute(wuv_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, GM_SMEM_ALLOC) == cudaSuccess;
        good &= cudaFuncSetAttribute(tail_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, TD_SMEM_ALLOC) == cudaSuccess;
        good &= cudaFuncSetAttribute(condense_prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, CP_SMEM_ALLOC) == cudaSuccess;
        good &= cudaFuncSetAttribute(attn_prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, AP_SMEM_ALLOC) == cudaSuccess;
        // One shared-memory carveout (the largest) for every kernel of the
        // decode chain, so that an SM moving from one kernel to the next of
        // a step need not change its L1 / shared-memory split.
        const auto carve = [](const void *k) {
            return cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout,
                                        int(cudaSharedmemCarveoutMaxShared)) == cudaSuccess;
        };
        good &= carve(reinterpret_cast<const void *>(attn_decode_kernel<MODE_MLA>));
        good &= carve(reinterpret_cast<const void *>(attn_decode_kernel<MODE_REPS>));
        good &= carve(reinterpret_cast<const void *>(attn_decode_kernel<MODE_LCA>));
        good &= carve(reinterpret_cast<const void *>(attn_decode_kernel<MODE_MLA, true>));
        good &= carve(reinterpret_cast<const void *>(attn_decode_kernel<MODE_LCA, true>));
        good &= carve(reinterpret_cast<const void *>(attn_decode_kernel<MODE_REPS, true>));
        good &= carve(reinterpret_cast<const void *>(tail_decode_kernel));
        good &= carve(reinterpret_cast<const void *>(prep_summary_kernel));
        good &= carve(reinterpret_cast<const void *>(append_token_kernel));
        good &= carve(reinterpret_cast<const void *>(condense_kernel<CdShape::kWarps, CdShape::kSlots>));
        if (!good) return LCA_ERR_CUDA;
        d.attrs_set = true;
    }
    *out = &d;
    return LCA_OK;
}

// ------------------------------------------------------------------ tensor maps
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int get_encode()
{
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_encode) return LCA_OK;
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
        return LCA_ERR_CUDA;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    return LCA_OK;
}

// 3-D bf16 map, dims {d0, d1, d2} (d0 innermost), byte strides {s1, s2},
// box {b0, b1, b2}, 128-byte swizzle, zero fill out of bounds.
int make_map3(CUtensorMap *m, const void *base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1,
              uint64_t s2, uint32_t b0, uint32_t b1, uint32_t b2)
{
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {s1, s2};
    cuuint32_t box[3] = {b0, b1, b2};
    cuuint32_t es[3] = {1, 1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
                          box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? LCA_OK : LCA_ERR_CUDA;
}

// Rows of 576 bf16 ([B][pitch][576]) as a 4-D tensor of 64-column chunks:
// (column within the chunk, row, chunk, sequence), so that one TMA box of
// [9 chunks][box_rows rows][64 columns] brings box_rows whole rows into
// shared memory in the layout of nine [rows x 64 columns] 128B-swizzled
// blocks, one per chunk.
int make_map_rows(CUtensorMap *m, const void *base, uint64_t rows, uint64_t B, uint64_t pitch_rows,
                  uint32_t box_rows)
{
    cuuint64_t dims[4] = {64, rows, LCA_D / 64, B};
    cuuint64_t strides[3] = {uint64_t(LCA_D) * 2, 128, pitch_rows * LCA_D * 2};
    cuuint32_t box[4] = {64, box_rows, LCA_D / 64, 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides,
                          box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? LCA_OK : LCA_ERR_CUDA;
}

// The prefill's group-major representatives [groups][nbc blocks][576] as a
// 4-D tensor (column within the chunk, block, group, chunk): a box of 64
// groups of one block lands as nine [64 groups x 64 columns] blocks.
int make_map_reps(CUtensorMap *m, const void *base, uint64_t nbc, uint64_t groups)
{
    cuuint64_t dims[4] = {64, nbc, groups, LCA_D / 64};
    cuuint64_t strides[3] = {uint64_t(LCA_D) * 2, nbc * LCA_D * 2, 128};
    cuuint32_t box[4] = {64, 1, 64, LCA_D / 64};
    cuuint32_t es[4] = {1, 1, 1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides,
                          box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? LCA_OK : LCA_ERR_CUDA;
}

// ------------------------------------------------------------------ timing / counting
struct ProfRec {
    cudaEvent_t a, b;
    int kid;
};
const char *kKernelNames[] = {"",         "prep_summary", "condense",    "attn_decode",      "combine_wuv",
                               "wuv_gemm", "attn_prefill", "condense_prefill", "selftest_wait", "append_token"};
constexpr int kNumKernelIds = 10;
bool g_prof_on = false;
std::vector<ProfRec> g_prof_used;
std::vector<std::pair<cudaEvent_t, cudaEvent_t>> g_prof_pool;
int64_t g_launches = 0;

struct Launch {
    cudaStream_t st;
    int kid;
    ProfRec rec{};
    bool timed = false;
    Launch(cudaStream_t s, int k) : st(s), kid(k)
    {
        std::lock_guard<std::mutex> lk(g_mu);
        ++g_launches;
        if (!g_prof_on) return;
        if (g_prof_pool.empty()) {
            cudaEvent_t x, y;
            if (cudaEventCreate(&x) != cudaSuccess) return;
            if (cudaEventCreate(&y) != cudaSuccess) { cudaEventDestroy(x); return; }
            g_prof_pool.push_back({x, y});
        }
        rec.a = g_prof_pool.back().first;
        rec.b = g_prof_pool.back().second;
        g_prof_pool.pop_back();
        rec.kid = k;
        timed = cudaEventRecord(rec.a, st) == cudaSuccess;
    }
    int done()
    {
        const cudaError_t e = cudaGetLastError();
        if (timed) {
            cudaEventRecord(rec.b, st);
            std::lock_guard<std::mutex> lk(g_mu);
            g_prof_used.push_back(rec);
        }
        return e == cudaSuccess ? LCA_OK : LCA_ERR_CUDA;
    }
};

// Launch with programmatic dependent launch allowed (the kernel may start
// its prologue while the previous kernel in the stream finishes; it calls
// griddepcontrol.wait before touching that kernel's results).
template <typename... KArgs, typename... Args>
cudaError_t launch_ex(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl,
                      Args &&...args)
{
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = pdl ? attr : nullptr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ------------------------------------------------------------------ workspace
struct DecodeWs {
    float *u;
    uint16_t *uhl;
    float *part_o;
    float *part_ml;
    uint16_t *o_bf16;
    int32_t *tile_start;   // [B+1], ragged batches only
    size_t bytes;
};

DecodeWs decode_ws_layout(void *ws, int B)
{
    DecodeWs w{};
    const size_t slots = size_t(kMaxCtas) + size_t(B);
    size_t off[7];
    off[0] = 0;
    off[1] = off[0] + align_up(size_t(B) * LCA_D * 4);                 // u
    off[2] = off[1] + align_up(size_t(B) * 2 * LCA_D * 2);             // uhl
    off[3] = off[2] + align_up(slots * LCA_HEADS * LCA_DC * 4);         // part_o
    off[4] = off[3] + align_up(slots * LCA_HEADS * 2 * 4);              // part_ml
    off[5] = off[4] + align_up(size_t(B) * LCA_HEADS * LCA_DC * 2);     // o_bf16
    off[6] = off[5] + align_up((size_t(B) + 1) * 4);                    // tile_start
    w.bytes = off[6];
    if (ws) {
        uint8_t *p = static_cast<uint8_t *>(ws);
        w.u = reinterpret_cast<float *>(p + off[0]);
        w.uhl = reinterpret_cast<uint16_t *>(p + off[1]);
        w.part_o = reinterpret_cast<float *>(p + off[2]);
        w.part_ml = reinterpret_cast<float *>(p + off[3]);
        w.o_bf16 = reinterpret_cast<uint16_t *>(p + off[4]);
        w.tile_start = reinterpret_cast<int32_t *>(p + off[5]);
    }
    return w;
}

// Blockwise prefill: summary queries of every block of the call, then one
// chunk of at most kPrefillChunk blocks at a time: its packed
// representatives and its bf16 attention output (the W_UV GEMM's A operand).
constexpr int64_t kPrefillChunk = 256;

struct PrefillWs {
    uint16_t *uhl;      // [B * nb][2][576]
    uint16_t *rep;      // [CP_G ceil(m_bound / CP_G)][chunk blocks][576]
    uint16_t *o_bf16;   // [chunk blocks * 16][16][512]
    size_t bytes;
};

PrefillWs prefill_ws_layout(void *ws, int B, int64_t nb, int64_t m_bound)
{
    PrefillWs w{};
    const int64_t nbc = std::min<int64_t>(nb, kPrefillChunk);
    size_t off[4];
    off[0] = 0;
    off[1] = off[0] + align_up(size_t(B) * size_t(nb) * 2 * LCA_D * 2);
    off[2] = off[1] + align_up(size_t(nbc) * size_t(CP_G * std::max<int64_t>((m_bound + CP_G - 1) / CP_G, 1)) *
                               LCA_D * 2);
    off[3] = off[2] + align_up(size_t(nbc) * 16 * LCA_HEADS * LCA_DC * 2);
    w.bytes = off[3];
    if (ws) {
        uint8_t *p = static_cast<uint8_t *>(ws);
        w.uhl = reinterpret_cast<uint16_t *>(p + off[0]);
        w.rep = reinterpret_cast<uint16_t *>(p + off[1]);
        w.o_bf16 = reinterpret_cast<uint16_t *>(p + off[2]);
    }
    return w;
}

bool params_ok(const lca_params &p)
{
    return p.g >= 1 && p.w >= 0 && std::isfinite(p.scale) && p.scale > 0.f && p.variant >= LCA_VARIANT_LCA &&
           p.variant <= LCA_VARIANT_SPARSE && p.cache_pitch >= 0;
}

// Rows between consecutive sequences of the cache (the packed layout when
// the caller leaves cache_pitch at 0), and whether it fits sequences of L rows.
int64_t cache_pitch(const lca_params &p, int64_t L) { return p.cache_pitch > 0 ? p.cache_pitch : L; }

bool pitch_ok(const lca_params &p, int B, int64_t L)
{
    const int64_t pitch = cache_pitch(p, L);
    return pitch >= L && int64_t(B) * pitch < (int64_t(1) << 40);
}

int64_t num_groups(int64_t L, const lca_params &p)
{
    if (!params_ok(p) || L <= p.w) return 0;
    return (L - p.w) / p.g;
}

// A pointer the kernels may dereference: device or managed memory, or pinned
// host memory mapped at the same address (cudaHostAlloc / cudaMallocHost /
// cudaHostRegister under unified addressing).  Pageable host memory and
// unknown addresses are refused before anything is launched.
int check_reachable(const void *p)
{
    cudaPointerAttributes at{};
    const cudaError_t e = cudaPointerGetAttributes(&at, p);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return (e == cudaErrorInvalidValue) ? LCA_ERR_INVALID_ARG : LCA_ERR_NO_DEVICE;
    }
    if (at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged) return LCA_OK;
    if (at.type == cudaMemoryTypeHost && at.devicePointer == p) return LCA_OK;
    return LCA_ERR_INVALID_ARG;
}

int check_common(const void *cache, const void *q, const void *w_uv, int B, int64_t L, float *out)
{
    if (!cache || !q || !w_uv || !out) return LCA_ERR_INVALID_ARG;
    if (B < 1 || L < 1 || L >= (int64_t(1) << 31) || int64_t(B) * L >= (int64_t(1) << 40)) return LCA_ERR_INVALID_ARG;
    if (!aligned16(cache) || !aligned16(q) || !aligned16(w_uv) || !aligned16(out)) return LCA_ERR_MISALIGNED;
    return LCA_OK;
}

int check_ws(void *ws, size_t ws_bytes, size_t need)
{
    if (!ws || ws_bytes < need) return LCA_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(ws) % kAlign) return LCA_ERR_MISALIGNED;
    return LCA_OK;
}

// Shared tail of the decode paths: split-L attention, combine, W_UV GEMM.
// Ragged batches (VARLEN): `lens` holds each sequence's length on the device,
// L and m are the largest length and its group count (the anchor row
// stride), and the tile offsets in w.tile_start were written by
// varlen_tiles_kernel just before; `window` is the local window w.
template <int MODE, bool VARLEN = false>
int run_attention(DeviceInfo *dev, const void *cache, const void *rep, const void *q, const void *w_uv, int B,
                  int64_t L, int64_t pitch, int64_t m, int64_t win0, float scale, float *out, float *o_lat,
                  int32_t *anchor,
                  const DecodeWs &w, cudaStream_t st, int64_t rep_stride = 0, float *lse_out = nullptr,
                  const int32_t *lens = nullptr, int window = 0)
{
    int rc = get_encode();
    if (rc) return rc;
    AttnArgs a{};
    a.q = static_cast<const uint16_t *>(q);
    a.uhl = w.uhl;
    a.L = L;
    a.m = m;
    a.win0 = win0;
    if (MODE == MODE_MLA) a.n_hist = 0;
    else if (MODE == MODE_REPS) a.n_hist = int((m + AT_TILE - 1) / AT_TILE);
    else a.n_hist = int((m + 3) / 4);
    a.n_tiles = a.n_hist + int((L - win0 + AT_TILE - 1) / AT_TILE);
    a.T = int64_t(B) * a.n_tiles;
    // a ragged batch's tile count is known on the device only: one CTA per
    // SM, each reading its range of the tile list
    a.G = int(std::min<int64_t>(std::min<int64_t>(dev->sms, kMaxCtas), VARLEN ? int64_t(kMaxCtas) : a.T));
    a.sl2 = scale * 1.4426950408889634f;
    a.part_o = w.part_o;
    a.part_ml = w.part_ml;
    a.anchor = anchor;
    a.lens = lens;
    a.tile_start = VARLEN ? w.tile_start : nullptr;
    a.B = B;
    a.w = window;
    a.after_prep = (!VARLEN && MODE == MODE_LCA && m > 0) ? 1 : 0;

    CUtensorMap map_cache, map_rep;
    rc = make_map_rows(&map_cache, cache, uint64_t(L), uint64_t(B), uint64_t(pitch), AT_TILE);
    if (rc) return rc;
    if (MODE == MODE_REPS && m > 0) {
        // rows per sequence: m, or the capacity of a representative cache
        const uint64_t stride_rows = uint64_t(rep_stride > 0 ? rep_stride : m);
        rc = make_map_rows(&map_rep, rep, uint64_t(m), uint64_t(B), stride_rows, AT_TILE);
        if (rc) return rc;
    } else {
        map_rep = map_cache;
    }
    {
        Launch l(st, K_ATTN);
        // the attention prologue overlaps the kernel before it: the
        // summary-query kernel (LCA; then the first cache loads too) or the
        // previous step's tail (the kernel waits for it before it reads any
        // input or writes a partial)
        const cudaError_t e = launch_ex(attn_decode_kernel<MODE, VARLEN>, dim3(a.G), dim3(AT_THREADS), AT_SMEM_ALLOC,
                                        st, true, map_cache, map_rep, a);
        if (e != cudaSuccess || (rc = l.done())) return LCA_ERR_CUDA;
    }
    CUtensorMap map_w = map_cache;   // unused when out is NULL (a shard's partial)
    if (out) rc = make_map3(&map_w, w_uv, LCA_DV, LCA_DC, LCA_HEADS, LCA_DV * 2, LCA_DC * LCA_DV * 2, 64, 64, 1);
    if (rc) return rc;
    {
        Launch l(st, K_COMBINE);
        // rows per CTA: enough CTAs (16 heads x row groups) to cover the SMs
        const int rpc = std::max(1, std::min(TD_ROWS, (LCA_HEADS * B + dev->sms - 1) / dev->sms));
        const cudaError_t e = launch_ex(tail_decode_kernel, dim3(LCA_HEADS, (B + rpc - 1) / rpc), dim3(256),
                                        TD_SMEM_ALLOC, st, true, map_w, (const float *)w.part_o,
                                        (const float *)w.part_ml, B, a.n_tiles, a.T, a.G, o_lat, out, rpc,
                                        lse_out, 0, int64_t(0), (const int32_t *)a.tile_start);
        if (e != cudaSuccess || (rc = l.done())) return LCA_ERR_CUDA;
    }
    return LCA_OK;
}

int launch_prep(const void *q_recent, int B, const lca_params &p, const DecodeWs &w, cudaStream_t st)
{
    Launch l(st, K_PREP);
    const float coef = p.scale / float(LCA_HEADS * p.g);
    const cudaError_t e = launch_ex(prep_summary_kernel, dim3(B, LCA_D / 64), dim3(PREP_THREADS), 0, st, true,
                                    static_cast<const uint16_t *>(q_recent), p.g, 1,
                                    int64_t(p.g) * LCA_HEADS * LCA_D, coef, w.u, w.uhl);
    if (e != cudaSuccess) return LCA_ERR_CUDA;
    return l.done();
}

// ------------------------------------------------------------------ no-allocation decode
// Scratch for lca_decode_noalloc lives in this module's own device memory, so
// a caller that cannot allocate (see include/lca.h) never has to.  It is
// sized for LCA_NOALLOC_MAX_BATCH sequences with the same layout as the
// caller-provided workspace of lca_decode; every GPU that loads the library
// keeps this array until the process exits.
constexpr size_t al256(size_t x) { return (x + 255) / 256 * 256; }
constexpr size_t noalloc_scratch_bytes(size_t B)
{
    return al256(B * LCA_D * 4) + al256(B * 2 * LCA_D * 2) + al256((kMaxCtas + B) * LCA_HEADS * LCA_DC * 4) +
           al256((kMaxCtas + B) * LCA_HEADS * 2 * 4) + al256(B * LCA_HEADS * LCA_DC * 2) + al256((B + 1) * 4);
}
constexpr size_t kNoAllocBytes = noalloc_scratch_bytes(LCA_NOALLOC_MAX_BATCH);

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

// Device address of g_noalloc_scratch on the current device, looked up once
// per device (the host-side symbol is only a stand-in and must never be
// handed to a kernel).
void *g_noalloc_ptr[64] = {};

int noalloc_scratch(void **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return LCA_ERR_NO_DEVICE;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return LCA_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return LCA_OK;
}

}  // namespace

// ====================================================================== C ABI
extern "C" {

int64_t lca_num_groups(int64_t L, lca_params p) { return num_groups(L, p); }

size_t lca_workspace_bytes(int op, int B, int64_t L, int64_t q_len, lca_params p)
{
    if (B < 1) return 0;
    switch (op) {
    case LCA_OP_MLA_DECODE:
    case LCA_OP_DECODE_ATTN:
    case LCA_OP_DECODE:
    case LCA_OP_CONDENSE:
        if (op != LCA_OP_MLA_DECODE && !params_ok(p)) return 0;
        return decode_ws_layout(nullptr, B).bytes;
    case LCA_OP_PREFILL: {
        if (!params_ok(p) || p.g != 16 || q_len < 16 || q_len % 16 || L < q_len) return 0;
        // the representatives of the last block a range inside [0, L) can hold
        const int cw = (p.w + 15) / 16;
        return prefill_ws_layout(nullptr, B, q_len / 16, pf_groups(L / 16 - 1, cw)).bytes;
    }
    default:
        return 0;
    }
}

int mla_decode_attn(const void *cache, const void *q, const void *w_uv, int B, int64_t L, float scale, float *out,
                    float *o_lat, void *ws, size_t ws_bytes, void *stream)
{
    int rc = check_common(cache, q, w_uv, B, L, out);
    if (rc) return rc;
    if (!std::isfinite(scale) || scale <= 0.f) return LCA_ERR_INVALID_ARG;
    if (o_lat && !aligned16(o_lat)) return LCA_ERR_MISALIGNED;
    const DecodeWs w = decode_ws_layout(ws, B);
    if ((rc = check_ws(ws, ws_bytes, w.bytes))) return rc;
    DeviceInfo *dev = nullptr;
    if ((rc = current_device(&dev)) || (rc = check_reachable(out))) return rc;   // out: device or pinned host
    return run_attention<MODE_MLA>(dev, cache, nullptr, q, w_uv, B, L, L, 0, 0, scale, out, o_lat, nullptr, w,
                                   static_cast<cudaStream_t>(stream));
}

int lca_condense(const void *cache, const void *q_recent, int B, int64_t L, lca_params p, void *rep,
                 int32_t *anchor, float *alpha, void *ws, size_t ws_bytes, void *stream)
{
    const int64_t m = num_groups(L, p);
    return lca_condense_append(cache, q_recent, B, L, p, 0, rep, m, anchor, alpha, ws, ws_bytes, stream);
}

int lca_condense_append(const void *cache, const void *q_recent, int B, int64_t L, lca_params p, int64_t j0,
                        void *rep, int64_t rep_cap, int32_t *anchor, float *alpha, void *ws, size_t ws_bytes,
                        void *stream)
{
    if (!cache || !q_recent) return LCA_ERR_INVALID_ARG;
    if (B < 1 || L < 1 || L >= (int64_t(1) << 31)) return LCA_ERR_INVALID_ARG;
    if (!params_ok(p) || !pitch_ok(p, B, L)) return LCA_ERR_INVALID_ARG;
    if (p.g != 16) return LCA_ERR_UNSUPPORTED;
    const int64_t m = num_groups(L, p);
    if (j0 < 0 || j0 > m || rep_cap < m) return LCA_ERR_INVALID_ARG;
    if (m > j0 && !rep) return LCA_ERR_INVALID_ARG;
    if (!aligned16(cache) || !aligned16(q_recent) || (rep && !aligned16(rep)) || (alpha && !aligned16(alpha)) ||
        (anchor && (reinterpret_cast<uintptr_t>(anchor) & 3u)))
        return LCA_ERR_MISALIGNED;
    const DecodeWs w = decode_ws_layout(ws, B);
    int rc = check_ws(ws, ws_bytes, w.bytes);
    if (rc) return rc;
    DeviceInfo *dev = nullptr;
    if ((rc = current_device(&dev))) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (m == j0) return LCA_OK;
    if ((rc = launch_prep(q_recent, B, p, w, st))) return rc;
    CondenseArgs a{};
    a.cache = static_cast<const uint16_t *>(cache);
    a.u = w.u;
    a.pitch = cache_pitch(p, L);
    a.m = m - j0;
    a.j0 = j0;
    a.stride = rep_cap;
    a.total = int64_t(B) * a.m;
    a.rep = static_cast<uint16_t *>(rep);
    a.anchor = anchor;
    a.alpha = alpha;
    a.variant = p.variant;
    const int64_t want = (a.total + CdShape::kWarps - 1) / CdShape::kWarps;
    const int grid = int(std::max<int64_t>(1, std::min<int64_t>(dev->sms, want)));
    Launch l(st, K_CONDENSE);
    if (launch_ex(condense_kernel<CdShape::kWarps, CdShape::kSlots>, dim3(grid), dim3(CdShape::kWarps * 32),
                  CdShape::kSmem, st, true, a) != cudaSuccess)
        return LCA_ERR_CUDA;
    return l.done();
}

int lca_decode_stored(const void *cache, const void *rep, int64_t rep_cap, const void *q, const void *w_uv, int B,
                      int64_t L, lca_params p, float *out, float *o_lat, void *ws, size_t ws_bytes, void *stream)
{
    int rc = check_common(cache, q, w_uv, B, L, out);
    if (rc) return rc;
    if (!params_ok(p) || !pitch_ok(p, B, L)) return LCA_ERR_INVALID_ARG;
    if (p.g != 16) return LCA_ERR_UNSUPPORTED;
    const int64_t m = num_groups(L, p);
    if (rep_cap < m || (m > 0 && !rep)) return LCA_ERR_INVALID_ARG;
    if ((rep && !aligned16(rep)) || (o_lat && !aligned16(o_lat))) return LCA_ERR_MISALIGNED;
    const DecodeWs w = decode_ws_layout(ws, B);
    if ((rc = check_ws(ws, ws_bytes, w.bytes))) return rc;
    DeviceInfo *dev = nullptr;
    if ((rc = current_device(&dev)) || (rc = check_reachable(out))) return rc;   // out: device or pinned host
    return run_attention<MODE_REPS>(dev, cache, rep, q, w_uv, B, L, cache_pitch(p, L), m, m * p.g, p.scale, out,
                                    o_lat, nullptr, w, static_cast<cudaStream_t>(stream), rep_cap);
}

int lca_decode_attn(const void *cache, const void *rep, const void *q, const void *w_uv, int B, int64_t L,
                    lca_params p, float *out, float *o_lat, void *ws, size_t ws_bytes, void *stream)
{
    int rc = check_common(cache, q, w_uv, B, L, out);
    if (rc) return rc;
    if (!params_ok(p) || !pitch_ok(p, B, L)) return LCA_ERR_INVALID_ARG;
    if (p.g != 16) return LCA_ERR_UNSUPPORTED;
    const int64_t m = num_groups(L, p);
    if (m > 0 && !rep) return LCA_ERR_INVALID_ARG;
    if ((rep && !aligned16(rep)) || (o_lat && !aligned16(o_lat))) return LCA_ERR_MISALIGNED;
    const DecodeWs w = decode_ws_layout(ws, B);
    if ((rc = check_ws(ws, ws_bytes, w.bytes))) return rc;
    DeviceInfo *dev = nullptr;
    if ((rc = current_device(&dev)) || (rc = check_reachable(out))) return rc;   // out: device or pinned host
    return run_attention<MODE_REPS>(dev, cache, rep, q, w_uv, B, L, cache_pitch(p, L), m, m * p.g, p.scale, out,
                                    o_lat, nullptr, w, static_cast<cudaStream_t>(stream));
}

int lca_decode(const void *cache, const void *q_recent, const void *q, const void *w_uv, int B, int64_t L,
               lca_params p, float *out, float *o_lat, int32_t *anchor, void *ws, size_t ws_bytes, void *stream)
{
    int rc = check_common(cache, q, w_uv, B, L, out);
    if (rc) return rc;
    if (!params_ok(p) || !pitch_ok(p, B, L)) return LCA_ERR_INVALID_ARG;
    if (p.variant != LCA_VARIANT_LCA) return LCA_ERR_UNSUPPORTED;   // ablations: lca_condense + lca_decode_attn
    if (p.g != 1 && p.g != 16) return LCA_ERR_UNSUPPORTED;
    if (p.g != 1 && !q_recent) return LCA_ERR_INVALID_ARG;
    if ((p.g != 1 && !aligned16(q_recent)) || (o_lat && !aligned16(o_lat)) ||
        (anchor && (reinterpret_cast<uintptr_t>(anchor) & 3u)))
        return LCA_ERR_MISALIGNED;
    const DecodeWs w = decode_ws_layout(ws, B);
    if ((rc = check_ws(ws, ws_bytes, w.bytes))) return rc;
    DeviceInfo *dev = nullptr;
    if ((rc = current_device(&dev)) || (rc = check_reachable(out))) return rc;   // out: device or pinned host
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t pitch = cache_pitch(p, L);
    if (p.g == 1)   // every token its own representative: MLA decode
        return run_attention<MODE_MLA>(dev, cache, nullptr, q, w_uv, B, L, pitch, 0, 0, p.scale, out, o_lat, nullptr,
                                       w, st);
    const int64_t m = num_groups(L, p);
    if (m > 0 && (rc = launch_prep(q_recent, B, p, w, st))) return rc;
    return run_attention<MODE_LCA>(dev, cache, nullptr, q, w_uv, B, L, pitch, m, m * p.g, p.scale, out, o_lat, anchor,
                                   w, st);
}

int lca_decode_varlen(const void *cache, const int32_t *lens, const void *q_recent, const void *q, const void *w_uv,
                      int B, int64_t L, lca_params p, float *out, float *o_lat, int32_t *anchor, void *ws,
                      size_t ws_bytes, void *stream)
{
    int rc = check_common(cache, q, w_uv, B, L, out);
    if (rc) return rc;
    if (!lens || !params_ok(p) || !pitch_ok(p, B, L)) return LCA_ERR_INVALID_ARG;
    if (p.variant != LCA_VARIANT_LCA) return LCA_ERR_UNSUPPORTED;
    if (p.g != 1 && p.g != 16) return LCA_ERR_UNSUPPORTED;
    if (p.g != 1 && !q_recent) return LCA_ERR_INVALID_ARG;
    // tile offsets are int32: the whole batch's tiles must stay below 2^31
    if (int64_t(B) * (L / AT_TILE + 2) >= (int64_t(1) << 31)) return LCA_ERR_UNSUPPORTED;
    if ((p.g != 1 && !aligned16(q_recent)) || (o_lat && !aligned16(o_lat)) ||
        (reinterpret_cast<uintptr_t>(lens) & 3u) || (anchor && (reinterpret_cast<uintptr_t>(anchor) & 3u)))
        return LCA_ERR_MISALIGNED;
    const DecodeWs w = decode_ws_layout(ws, B);
    if ((rc = check_ws(ws, ws_bytes, w.bytes))) return rc;
    DeviceInfo *dev = nullptr;
    if ((rc = current_device(&dev)) || (rc = check_reachable(out))) return rc;   // out: device or pinned host
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t pitch = cache_pitch(p, L);
    {
        Launch l(st, K_PREP);
        if (p.g == 1)
            varlen_tiles_kernel<MODE_MLA><<<1, VT_THREADS, 0, st>>>(lens, B, L, p.w, w.tile_start);
        else
            varlen_tiles_kernel<MODE_LCA><<<1, VT_THREADS, 0, st>>>(lens, B, L, p.w, w.tile_start);
        if ((rc = l.done())) return rc;
    }
    if (p.g == 1)
        return run_attention<MODE_MLA, true>(dev, cache, nullptr, q, w_uv, B, L, pitch, 0, 0, p.scale, out, o_lat,
                                             nullptr, w, st, 0, nullptr, lens, p.w);
    const int64_t m = num_groups(L, p);   // the anchor row stride
    if ((rc = launch_prep(q_recent, B, p, w, st))) return rc;
    return run_attention<MODE_LCA, true>(dev, cache, nullptr, q, w_uv, B, L, pitch, m, m * p.g, p.scale, out, o_lat,
                                         anchor, w, st, 0, nullptr, lens, p.w);
}

int lca_decode_stored_varlen(const void *cache, const void *rep, int64_t rep_cap, const int32_t *lens, const void *q,
                             const void *w_uv, int B, int64_t L, lca_params p, float *out, float *o_lat, void *ws,
                             size_t ws_bytes, void *stream)
{
    int rc = check_common(cache, q, w_uv, B, L, out);
    if (rc) return rc;
    if (!lens || !params_ok(p) || !pitch_ok(p, B, L)) return LCA_ERR_INVALID_ARG;
    if (p.g != 16) return LCA_ERR_UNSUPPORTED;
    const int64_t m = num_groups(L, p);   // the longest sequence's groups
    if (rep_cap < m || (m > 0 && !rep)) return LCA_ERR_INVALID_ARG;
    if (int64_t(B) * (L / AT_TILE + 2) >= (int64_t(1) << 31)) return LCA_ERR_UNSUPPORTED;
    if ((rep && !aligned16(rep)) || (o_lat && !aligned16(o_lat)) || (reinterpret_cast<uintptr_t>(lens) & 3u))
        return LCA_ERR_MISALIGNED;
    const DecodeWs w = decode_ws_layout(ws, B);
    if ((rc = check_ws(ws, ws_bytes, w.bytes))) return rc;
    DeviceInfo *dev = nullptr;
    if ((rc = current_device(&dev)) || (rc = check_reachable(out))) return rc;   // out: device or pinned host
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    {
        Launch l(st, K_PREP);
        varlen_tiles_kernel<MODE_REPS><<<1, VT_THREADS, 0, st>>>(lens, B, L, p.w, w.tile_start);
        if ((rc = l.done())) return rc;
    }
    return run_attention<MODE_REPS, true>(dev, cache, rep, q, w_uv, B, L, cache_pitch(p, L), m, m * p.g, p.scale,
                                          out, o_lat, nullptr, w, st, rep_cap, nullptr, lens, p.w);
}

int lca_decode_noalloc(const void *cache, const void *q_recent, const void *q, const void *w_uv, int B, int64_t L,
                       lca_params p, float *out, float *o_lat, int32_t *anchor, void *stream)
{
    int rc = check_common(cache, q, w_uv, B, L, out);
    if (rc) return rc;
    if (!params_ok(p) || !pitch_ok(p, B, L)) return LCA_ERR_INVALID_ARG;
    if (p.variant != LCA_VARIANT_LCA) return LCA_ERR_UNSUPPORTED;
    if (B > LCA_NOALLOC_MAX_BATCH) return LCA_ERR_SCRATCH_LIMIT;
    if (p.g != 1 && p.g != 16) return LCA_ERR_UNSUPPORTED;
    if (p.g != 1 && !q_recent) return LCA_ERR_INVALID_ARG;
    if ((q_recent && !aligned16(q_recent)) || (o_lat && !aligned16(o_lat)) ||
        (anchor && (reinterpret_cast<uintptr_t>(anchor) & 3u)))
        return LCA_ERR_MISALIGNED;
    void *scratch = nullptr;
    if ((rc = noalloc_scratch(&scratch))) return rc;
    const DecodeWs w = decode_ws_layout(scratch, B);
    if (w.bytes > kNoAllocBytes) return LCA_ERR_SCRATCH_LIMIT;
    DeviceInfo *dev = nullptr;
    if ((rc = current_device(&dev)) || (rc = check_reachable(out))) return rc;   // out: device or pinned host
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t pitch = cache_pitch(p, L);
    if (p.g == 1)
        return run_attention<MODE_MLA>(dev, cache, nullptr, q, w_uv, B, L, pitch, 0, 0, p.scale, out, o_lat, nullptr,
                                       w, st);
    const int64_t m = num_groups(L, p);
    if (m > 0 && (rc = launch_prep(q_recent, B, p, w, st))) return rc;
    return run_attention<MODE_LCA>(dev, cache, nullptr, q, w_uv, B, L, pitch, m, m * p.g, p.scale, out, o_lat, anchor,
                                   w, st);
}

int lca_decode_shard(const void *cache_shard, const void *q_recent, const void *q, int B, int64_t L, int64_t row0,
                     int64_t L_shard, lca_params p, float *part, int32_t *anchor, void *ws, size_t ws_bytes,
                     void *stream)
{
    if (!cache_shard || !q || !part) return LCA_ERR_INVALID_ARG;
    if (B < 1 || L < 1 || L >= (int64_t(1) << 31) || L_shard < 1 || row0 < 0 || row0 + L_shard > L ||
        int64_t(B) * L_shard >= (int64_t(1) << 40))
        return LCA_ERR_INVALID_ARG;
    if (!params_ok(p) || !pitch_ok(p, B, L_shard)) return LCA_ERR_INVALID_ARG;
    if (p.g != 16 || p.variant != LCA_VARIANT_LCA) return LCA_ERR_UNSUPPORTED;
    const int64_t m = num_groups(L, p), hist_end = m * p.g, row1 = row0 + L_shard;
    // whole groups; a shard that does not reach L lies inside the history,
    // so the window belongs to the last shard alone
    if (row0 % p.g || row0 > hist_end || (row1 < L && (row1 % p.g || row1 > hist_end))) return LCA_ERR_INVALID_ARG;
    const int64_t m_loc = (std::min(row1, hist_end) - row0) / p.g;
    if (m_loc > 0 && !q_recent) return LCA_ERR_INVALID_ARG;
    if (!aligned16(cache_shard) || !aligned16(q) || !aligned16(part) || (q_recent && !aligned16(q_recent)) ||
        (anchor && (reinterpret_cast<uintptr_t>(anchor) & 3u)))
        return LCA_ERR_MISALIGNED;
    int rc = LCA_OK;
    const DecodeWs w = decode_ws_layout(ws, B);
    if ((rc = check_ws(ws, ws_bytes, w.bytes))) return rc;
    DeviceInfo *dev = nullptr;
    if ((rc = current_device(&dev))) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (m_loc > 0 && (rc = launch_prep(q_recent, B, p, w, st))) return rc;
    // the shard is an LCA decode of its own L_shard rows: m_loc groups, then
    // (last shard only) the window; o and lse2 go to the partial record
    float *lse = part + size_t(B) * LCA_HEADS * LCA_DC;
    return run_attention<MODE_LCA>(dev, cache_shard, nullptr, q, nullptr, B, L_shard, cache_pitch(p, L_shard), m_loc,
                                   m_loc * p.g, p.scale, nullptr, part, anchor, w, st, 0, lse);
}

int lca_combine_shards(const float *parts, int n_shards, int B, const void *w_uv, float *out, float *o_lat,
                       void *stream)
{
    if (!parts || !w_uv || !out || n_shards < 1 || B < 1 || B > (1 << 20)) return LCA_ERR_INVALID_ARG;
    if (!aligned16(parts) || !aligned16(w_uv) || !aligned16(out) || (o_lat && !aligned16(o_lat)))
        return LCA_ERR_MISALIGNED;
    int rc = get_encode();
    if (rc) return rc;
    DeviceInfo *dev = nullptr;
    if ((rc = current_device(&dev)) || (rc = check_reachable(out))) return rc;   // out: device or pinned host
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    CUtensorMap map_w;
    rc = make_map3(&map_w, w_uv, LCA_DV, LCA_DC, LCA_HEADS, LCA_DV * 2, LCA_DC * LCA_DV * 2, 64, 64, 1);
    if (rc) return rc;
    Launch l(st, K_COMBINE);
    const int rpc = std::max(1, std::min(TD_ROWS, (LCA_HEADS * B + dev->sms - 1) / dev->sms));
    const int64_t stride = int64_t(B) * LCA_HEADS * LCA_SHARD_RECORD_PER_HEAD;
    const cudaError_t e = launch_ex(tail_decode_kernel, dim3(LCA_HEADS, (B + rpc - 1) / rpc), dim3(256),
                                    TD_SMEM_ALLOC, st, false, map_w, parts, (const float *)nullptr, B, 0,
                                    int64_t(0), 0, o_lat, out, rpc, (float *)nullptr, n_shards, stride,
                                    (const int32_t *)nullptr);
    if (e != cudaSuccess || (rc = l.done())) return LCA_ERR_CUDA;
    return LCA_OK;
}

int lca_prefill_block(const void *cache, const void *q, const void *w_uv, int B, int64_t L, int64_t q_start,
                      int64_t q_len, lca_params p, float *out, float *o_lat, int32_t *anchor, void *ws,
                      size_t ws_bytes, void *stream)
{
    int rc = check_common(cache, q, w_uv, B, L, out);
    if (rc) return rc;
    if (!params_ok(p) || !pitch_ok(p, B, L)) return LCA_ERR_INVALID_ARG;
    if (p.g != 16) return LCA_ERR_UNSUPPORTED;
    if (q_start < 0 || q_len < 0 || q_start % 16 || q_len % 16 || q_start + q_len > L) return LCA_ERR_INVALID_ARG;
    if (L > (int64_t(1) << 27)) return LCA_ERR_UNSUPPORTED;   // query rows 16 L index a TMA map
    if (int64_t(B) * (q_len / 16) >= (int64_t(1) << 31)) return LCA_ERR_UNSUPPORTED;   // block index of a TMA map
    if ((o_lat && !aligned16(o_lat)) || (anchor && (reinterpret_cast<uintptr_t>(anchor) & 3u)))
        return LCA_ERR_MISALIGNED;
    if (q_len == 0) return LCA_OK;
    const int cw = (p.w + 15) / 16;
    const int64_t k0 = q_start / 16, nb = q_len / 16;
    const int64_t m_ld = pf_groups(k0 + nb - 1, cw);   // groups of the last block: anchor row length
    const PrefillWs w = prefill_ws_layout(ws, B, nb, m_ld);
    if ((rc = check_ws(ws, ws_bytes, w.bytes))) return rc;
    DeviceInfo *dev = nullptr;
    if ((rc = current_device(&dev)) || (rc = check_reachable(out))) return rc;   // out: device or pinned host
    if ((rc = get_encode())) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const uint16_t *qv = static_cast<const uint16_t *>(q);

    CUtensorMap map_cache, map_rows, map_q, map_u, map_w;
    const uint64_t seq_bytes = uint64_t(cache_pitch(p, L)) * LCA_D * 2;
    if ((rc = make_map_rows(&map_cache, cache, uint64_t(L), uint64_t(B), uint64_t(cache_pitch(p, L)), 64)))
        return rc;
    // the condensation's history tiles: CP_ROWS rows
    if ((rc = make_map3(&map_rows, cache, LCA_D, uint64_t(L), uint64_t(B), uint64_t(LCA_D) * 2, seq_bytes, 64,
                        CP_ROWS, 1)))
        return rc;
    if ((rc = make_map_rows(&map_q, q, uint64_t(L) * LCA_HEADS, uint64_t(B), uint64_t(L) * LCA_HEADS, 64)))
        return rc;
    if ((rc = make_map3(&map_u, w.uhl, LCA_D, 2, uint64_t(B) * uint64_t(nb), uint64_t(LCA_D) * 2,
                        uint64_t(LCA_D) * 4, 64, 1, 128)))
        return rc;
    if ((rc = make_map3(&map_w, w_uv, LCA_DV, LCA_DC, LCA_HEADS, LCA_DV * 2, LCA_DC * LCA_DV * 2, 64, 64, 1)))
        return rc;

    // summary query of every block (mean of its own 16 queries, folded)
    {
        Launch l(st, K_PREP);
        const float coef = p.scale / float(LCA_HEADS * 16);
        const cudaError_t e = launch_ex(prep_summary_kernel, dim3(unsigned(int64_t(B) * nb), LCA_D / 64),
                                        dim3(PREP_THREADS), 0, st, false, qv + size_t(k0) * 16 * LCA_HEADS * LCA_D,
                                        16, int(nb), int64_t(L) * LCA_HEADS * LCA_D, coef, (float *)nullptr, w.uhl);
        if (e != cudaSuccess || (rc = l.done())) return LCA_ERR_CUDA;
    }
    const float sl2 = p.scale * 1.4426950408889634f;
    for (int b = 0; b < B; ++b) {
        for (int64_t kc0 = k0; kc0 < k0 + nb; kc0 += kPrefillChunk) {
            const int nbc = int(std::min<int64_t>(kPrefillChunk, k0 + nb - kc0));
            const int n_gt = int((pf_groups(kc0 + nbc - 1, cw) + CP_G - 1) / CP_G);   // group tiles of the chunk
            CUtensorMap map_rep = map_cache;
            if (n_gt > 0) {
                // group-major [CP_G n_gt][nbc][576]; a box is 64 groups of one block
                if ((rc = make_map_reps(&map_rep, w.rep, uint64_t(nbc), uint64_t(CP_G) * n_gt)))
                    return rc;
                CondPreArgs c{};
                c.kc0 = kc0;
                c.nbc = nbc;
                c.cw = cw;
                c.b = b;
                c.n_gt = n_gt;
                c.ublk0 = int(int64_t(b) * nb + (kc0 - k0));
                c.rep = w.rep;
                c.k0 = k0;
                c.m_ld = m_ld;
                c.anchor = anchor ? anchor + size_t(b) * size_t(nb) * size_t(m_ld) : nullptr;
                c.variant = p.variant;
                const int n_bt = (nbc + 127) / 128;
                Launch l(st, K_PREFILL_CONDENSE);
                const cudaError_t e = launch_ex(condense_prefill_kernel, dim3(unsigned(n_bt * c.n_gt)),
                                                dim3(CP_THREADS), CP_SMEM_ALLOC, st, false, map_rows, map_u, c);
                if (e != cudaSuccess || (rc = l.done())) return LCA_ERR_CUDA;
            }
            const size_t row_out = size_t(b) * size_t(q_len) + size_t(16 * (kc0 - k0));   // first output row
            {
                AttnPreArgs a{};
                a.L = L;
                a.b = b;
                a.kc0 = kc0;
                a.nbc = nbc;
                a.cw = cw;
                a.sl2 = sl2;
                a.o_bf16 = w.o_bf16;
                a.o_lat = o_lat ? o_lat + row_out * LCA_HEADS * LCA_DC : nullptr;
                Launch l(st, K_PREFILL);
                const cudaError_t e = launch_ex(attn_prefill_kernel, dim3(unsigned(4 * nbc)), dim3(AP_THREADS),
                                                AP_SMEM_ALLOC, st, false, map_cache, map_q, map_rep, a);
                if (e != cudaSuccess || (rc = l.done())) return LCA_ERR_CUDA;
            }
            {
                const int64_t R = int64_t(16) * nbc;
                CUtensorMap map_a;
                if ((rc = make_map3(&map_a, w.o_bf16, LCA_DC, LCA_HEADS, uint64_t(R), uint64_t(LCA_DC) * 2,
                                    uint64_t(LCA_HEADS) * LCA_DC * 2, 64, 1, 128)))
                    return rc;
                Launch l(st, K_GEMM);
                const cudaError_t e = launch_ex(wuv_gemm_kernel, dim3(unsigned((R + 127) / 128), LCA_HEADS),
                                                dim3(128), GM_SMEM_ALLOC, st, false, map_a, map_w,
                                                out + row_out * LCA_HEADS * LCA_DV, R);
                if (e != cudaSuccess || (rc = l.done())) return LCA_ERR_CUDA;
            }
        }
    }
    return LCA_OK;
}

int lca_append_token(const void *rows, void *cache, int B, int64_t pitch, int64_t pos, const void *q, void *ring,
                     int g, int slot, void *q_dst, void *stream)
{
    if (!rows || !cache || B < 1 || pitch < 1 || pos < 0 || pos >= pitch) return LCA_ERR_INVALID_ARG;
    if (int64_t(B) * pitch >= (int64_t(1) << 40)) return LCA_ERR_INVALID_ARG;
    if ((q == nullptr) != (ring == nullptr) || (q_dst && !q)) return LCA_ERR_INVALID_ARG;
    if (q && (g < 1 || slot < 0 || slot >= g)) return LCA_ERR_INVALID_ARG;
    if (!aligned16(rows) || !aligned16(cache) || (q && (!aligned16(q) || !aligned16(ring))) ||
        (q_dst && !aligned16(q_dst)))
        return LCA_ERR_MISALIGNED;
    DeviceInfo *dev = nullptr;
    int rc = current_device(&dev);
    if (rc) return rc;
    for (const void *p : {rows, static_cast<const void *>(cache), q, static_cast<const void *>(ring),
                          static_cast<const void *>(q_dst)})
        if (p && (rc = check_reachable(p))) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    Launch l(st, K_APPEND);
    const cudaError_t e = launch_ex(append_token_kernel, dim3(B, APPEND_SPLIT), dim3(APPEND_THREADS), 0, st, true,
                                    static_cast<const uint4 *>(rows), static_cast<uint4 *>(cache), pitch, pos,
                                    static_cast<const uint4 *>(q), static_cast<uint4 *>(ring), g, slot,
                                    static_cast<uint4 *>(q_dst));
    if (e != cudaSuccess) return LCA_ERR_CUDA;
    return l.done();
}

int lca_selftest_wait_timeout(void *stream)
{
    int rc = LCA_OK;
    DeviceInfo *dev = nullptr;
    if ((rc = current_device(&dev))) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    Launch l(st, K_SELFTEST);
    selftest_wait_kernel<<<1, 32, 0, st>>>();
    return l.done();
}

const char *lca_strerror(int status)
{
    switch (status) {
    case LCA_OK: return "ok";
    case LCA_ERR_INVALID_ARG: return "invalid argument";
    case LCA_ERR_MISALIGNED: return "pointer not aligned (16 bytes; workspace 256)";
    case LCA_ERR_WORKSPACE: return "workspace missing or too small";
    case LCA_ERR_UNSUPPORTED: return "parameter not supported by these kernels";
    case LCA_ERR_CUDA: return "CUDA call or kernel launch failed";
    case LCA_ERR_NO_DEVICE: return "current device is not an sm_100 GPU";
    case LCA_ERR_DEVICE_TIMEOUT: return "a kernel's bounded wait expired";
    case LCA_ERR_SCRATCH_LIMIT: return "batch larger than the built-in scratch of lca_decode_noalloc allows";
    default: return "unknown status";
    }
}

int lca_device_status(int clear, int *detail)
{
    int v = 0;
    if (cudaDeviceSynchronize() != cudaSuccess) return LCA_ERR_CUDA;
    if (cudaMemcpyFromSymbol(&v, lca::g_status, sizeof v) != cudaSuccess) return LCA_ERR_CUDA;
    if (clear) {
        const int z = 0;
        if (cudaMemcpyToSymbol(lca::g_status, &z, sizeof z) != cudaSuccess) return LCA_ERR_CUDA;
    }
    if (detail) *detail = v;
    return v == 0 ? LCA_OK : LCA_ERR_DEVICE_TIMEOUT;
}

int lca_profile_enable(int on)
{
    std::lock_guard<std::mutex> lk(g_mu);
    g_prof_on = on != 0;
    return LCA_OK;
}

int lca_profile_collect(lca_kernel_time *out, int max)
{
    std::vector<ProfRec> recs;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        recs.swap(g_prof_used);
    }
    lca_kernel_time acc[kNumKernelIds];
    std::memset(acc, 0, sizeof acc);
    int rc = LCA_OK;
    for (const ProfRec &r : recs) {
        float ms = 0.f;
        if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess)
            rc = LCA_ERR_CUDA;
        acc[r.kid].launches += 1;
        acc[r.kid].total_ms += ms;
    }
    {
        std::lock_guard<std::mutex> lk(g_mu);
        for (const ProfRec &r : recs) g_prof_pool.push_back({r.a, r.b});
    }
    if (rc) return rc;
    int n = 0;
    for (int k = 1; k < kNumKernelIds && n < max; ++k) {
        if (!acc[k].launches) continue;
        std::snprintf(out[n].name, sizeof out[n].name, "%s", kKernelNames[k]);
        out[n].launches = acc[k].launches;
        out[n].total_ms = acc[k].total_ms;
        ++n;
    }
    return n;
}

int64_t lca_launch_count(void)
{
    std::lock_guard<std::mutex> lk(g_mu);
    return g_launches;
}

}  // extern "C"

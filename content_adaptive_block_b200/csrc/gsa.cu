// libgsa: the C ABI of include/gsa.h.  Host-side argument checks, TMA
// descriptor set-up and kernel launches; all arithmetic of the path runs in
// the kernels included below.  One translation unit, so the device error
// word is a single symbol.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>
#include <mutex>

#include "gsa.h"

#include "common.cuh"
#include "deflate_lane.cuh"
#include "flags_csr.cuh"
#include "mask_pipeline.cuh"
#include "fixed_csr.cuh"

static_assert(GSA_MAX_FIXED_BLOCKS == gsa::fixed::kMaxBlocks, "header and kernel agree");
static_assert(GSA_MAX_RANDOM_BLOCKS == gsa::fixed::kMaxRandom, "header and kernel agree");
#include "attn_fwd_f32.cuh"
#include "attn_fwd_bf16.cuh"
#include "attn_bwd_bf16.cuh"
#include "gemm.cuh"

namespace {

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

gsa_status launch_status() {
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? GSA_OK : GSA_ERR_CUDA;
}

// ---- scratch of gsa_attn_bwd_noalloc
//
// Some callers cannot allocate device memory themselves (a host framework
// that owns every byte through its own pool, or a latency-bound loop that
// cannot afford cudaMalloc's implicit synchronisation).  For them the
// backward's per-row scratch (D_t = dO_t · O_t, float32) lives in this
// fixed array, which every GPU that loads the library holds until exit.
constexpr int64_t kNoAllocRows = int64_t(1) << 21;   // query rows (B*H*L); 16 MiB
static __device__ __align__(256) float g_bwd_noalloc_scratch[2 * kNoAllocRows + 64];   // D, LSE log2(e), counters
constexpr int kMaxDevices = 64;

// Device address of the scratch array on the current device, looked up once
// per device (host code cannot use the symbol itself as an address).
float* noalloc_scratch(gsa_status* st) {
    static std::mutex mu;
    static float* addr[kMaxDevices] = {};
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        *st = GSA_ERR_CUDA;
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_bwd_noalloc_scratch) != cudaSuccess || !p) {
            *st = GSA_ERR_CUDA;
            return nullptr;
        }
        addr[dev] = static_cast<float*>(p);
    }
    *st = GSA_OK;
    return addr[dev];
}

// ---- work counters of the persistent forward
//
// The forward takes no workspace, so its persistent kernel draws items from
// one of these slots (work counter, CTAs finished), a different slot per
// launch in turn; the launch's last CTA returns its slot to zero.  Up to
// kFwdSlots forward launches may therefore be in flight at once.
constexpr int kFwdSlots = 256;
static __device__ int g_fwd_tickets[2 * kFwdSlots];

int* fwd_ticket_slot() {
    static std::mutex mu;
    static int* addr[kMaxDevices] = {};
    static unsigned next[kMaxDevices] = {};
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_fwd_tickets) != cudaSuccess || !p) return nullptr;
        addr[dev] = static_cast<int*>(p);
    }
    const unsigned slot = next[dev]++ % kFwdSlots;
    return addr[dev] + 2 * slot;
}

bool csr_ok(const gsa_block_csr* c) {
    return c && c->B >= 1 && c->nblk >= 1 && c->row_ptr && c->col_idx && c->col_ptr && c->row_idx && c->q_order &&
           c->k_order && c->capacity >= gsa_csr_capacity(c->nblk);
}

// Common checks of an attention call; fills the class table.
inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The tensors' layouts: dense [B][H][L][d] without desc->layout; with it,
// strides that are positive multiples of 8 elements (16 bytes, as TMA
// requires) with each token's d values inside one stride step.
gsa_status resolve_layout(const gsa_attn_desc* d, gsa::TokLayout* lq, gsa::TokLayout* lo) {
    const int64_t dense_h = d->L * d->d, dense_s = d->H * dense_h;
    if (!d->layout) {
        *lq = *lo = gsa::TokLayout{dense_s, dense_h, d->d};
        return GSA_OK;
    }
    const gsa_attn_layout& y = *d->layout;
    const int64_t st[6] = {y.qkv_s, y.qkv_h, y.qkv_l, y.o_s, y.o_h, y.o_l};
    for (int64_t s : st)
        if (s <= 0 || s % 8 != 0) return GSA_ERR_INVALID_ARGUMENT;
    if (y.qkv_l < d->d || y.o_l < d->d) return GSA_ERR_INVALID_ARGUMENT;
    *lq = gsa::TokLayout{y.qkv_s, y.qkv_h, y.qkv_l};
    *lo = gsa::TokLayout{y.o_s, y.o_h, y.o_l};
    return GSA_OK;
}

template <int D, bool K4>
gsa_status launch_fwd(dim3 grid, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                      const gsa::bf16::FwdParams& p, cudaStream_t cs) {
    using C = gsa::bf16::FwdCfg<D>;
    if (!gsa::smem_opt_in(gsa::bf16::attn_fwd_bf16_kernel<D, K4>, C::kSmemBytes)) return GSA_ERR_CUDA;
    gsa::bf16::attn_fwd_bf16_kernel<D, K4><<<grid, gsa::bf16::FwdShape<D>::kThreads, C::kSmemBytes, cs>>>(tq, tk, tv,
                                                                                                        p);
    return launch_status();
}

// The persistent forward: as many CTAs as fit on the device at once (two per
// SM at d = 64, one at d = 128), at most one per work item.
template <int D, bool K4>
gsa_status launch_fwd_persist(int64_t items, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                              const gsa::bf16::FwdParams& p, cudaStream_t cs) {
    using C = gsa::bf16::FwdPCfg<D>;
    if (!gsa::smem_opt_in(gsa::bf16::attn_fwd_persist_kernel<D, K4>, C::kSmemBytes)) return GSA_ERR_CUDA;
    const int64_t full = static_cast<int64_t>(C::kCtasPerSm) * gsa::bwd::sm_count();
    const unsigned ctas = static_cast<unsigned>(items < full ? items : full);
    gsa::bf16::attn_fwd_persist_kernel<D, K4><<<ctas, C::kThreads, C::kSmemBytes, cs>>>(tq, tk, tv, p);
    return launch_status();
}

// The lengths kernel for blocks of at most MAXB bytes: 32 blocks per warp,
// one per lane.
template <int MAXB>
gsa_status launch_lengths_lane(const uint8_t* bytes, int b, int64_t total, int32_t* lengths, cudaStream_t cs) {
    using K = gsa::deflate_lane::KernelShape<MAXB>;
    const int bpw = gsa::deflate_lane::blocks_per_warp(total, static_cast<int64_t>(gsa::bwd::sm_count()) * K::kResident);
    const int64_t per_cta = static_cast<int64_t>(bpw) * K::kWarps;
    const int64_t grid = (total + per_cta - 1) / per_cta;
    if (grid > 0x7fffffff) return GSA_ERR_UNSUPPORTED;
    if (!gsa::smem_opt_in(gsa::deflate_lane::block_lengths_lane_kernel<MAXB>, K::kSmemBytes)) return GSA_ERR_CUDA;
    gsa::deflate_lane::block_lengths_lane_kernel<MAXB><<<static_cast<unsigned>(grid), 32 * K::kWarps, K::kSmemBytes,
                                                         cs>>>(bytes, b, total, bpw, lengths);
    return launch_status();
}

// The one-launch mask stage for blocks of at most MAXB bytes on CTAs of T
// warps (W of them computing lengths): a cooperative launch (every CTA
// resident: the phases meet at a grid barrier) of as many CTAs as fit on the
// device at once, or fewer when the batch has fewer chunks and list jobs.
template <int MAXB, int W, int T>
gsa_status launch_pipeline_shape(const gsa::pipeline::PipeArgs& P, cudaStream_t cs) {
    using S = gsa::pipeline::Shape<MAXB, W, T>;
    auto kernel = gsa::pipeline::mask_pipeline_kernel<MAXB, W, T>;
    if (!gsa::smem_opt_in(kernel, static_cast<int>(S::kSmemBytes))) return GSA_ERR_CUDA;
    int per_sm = 0;
    const int sms = gsa::bwd::sm_count();
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, 32 * T, S::kSmemBytes) != cudaSuccess ||
        per_sm < 1 || sms < 1)
        return GSA_ERR_CUDA;
    gsa::pipeline::PipeArgs Q = P;
    Q.bpw = gsa::deflate_lane::blocks_per_warp(P.total, static_cast<int64_t>(per_sm) * sms * W);
    const int64_t chunks = (P.total + Q.bpw - 1) / Q.bpw;
    const int64_t njobs = static_cast<int64_t>(P.B) * (P.nper > 0 ? P.nper : 1);
    int64_t grid = static_cast<int64_t>(per_sm) * sms;
    // a list job per warp for short lists when there are more jobs than CTAs
    // (measured faster up to 64 blocks per sample; longer lists go faster
    // with a CTA's warps on each job)
    Q.warp_jobs = P.nblk <= S::kMaxWarpJobBlocks && njobs > grid ? 1 : 0;
    const int64_t jobs = Q.warp_jobs ? (njobs + T - 1) / T : njobs;
    const int64_t want = chunks > jobs ? chunks : jobs;   // a chunk per CTA where possible: spread over the SMs
    if (want < grid) grid = want;
    void* args[] = {&Q};
    const cudaError_t e = cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(kernel),
                                                      dim3(static_cast<unsigned>(grid)), dim3(32 * T), args,
                                                      S::kSmemBytes, cs);
    return e == cudaSuccess ? GSA_OK : GSA_ERR_CUDA;
}

// Many short list jobs (more than one per SM, at most 128 blocks a sample)
// run on the narrow CTAs, one job per CTA side by side; a few jobs, or long
// lists, run on the wide ones, each job with 32 warps (measured over 256
// samples: the narrow shape 8-10 % faster at 64 blocks a sample and 0-4 % at
// 128, the wide one 15-19 % faster at 256).
template <int MAXB>
gsa_status launch_pipeline(const gsa::pipeline::PipeArgs& P, cudaStream_t cs) {
    using SS = gsa::pipeline::Shapes<MAXB>;
    const int64_t njobs = static_cast<int64_t>(P.B) * (P.nper > 0 ? P.nper : 1);
    if (njobs > gsa::bwd::sm_count() && P.nblk <= 128)
        return launch_pipeline_shape<MAXB, SS::kNarrowW, SS::kNarrowT>(P, cs);
    return launch_pipeline_shape<MAXB, SS::kWideW, SS::kWideT>(P, cs);
}

gsa_status check_attn(const gsa_attn_desc* d, const gsa_block_csr* csr, uint8_t* cls) {
    if (!d || !csr || !d->head_classes) return GSA_ERR_INVALID_ARGUMENT;
    if (!csr_ok(csr)) return csr && csr->capacity < gsa_csr_capacity(csr->nblk) ? GSA_ERR_CAPACITY
                                                                              : GSA_ERR_INVALID_ARGUMENT;
    if (d->B < 1 || d->H < 1 || d->L < 1 || d->b < 1 || d->d < 1) return GSA_ERR_INVALID_ARGUMENT;
    if (d->H > GSA_MAX_HEADS) return GSA_ERR_UNSUPPORTED;
    if (d->B != csr->B || d->L != static_cast<int64_t>(csr->nblk) * d->b) return GSA_ERR_INVALID_ARGUMENT;
    if (!(d->scale >= 0.f) || !std::isfinite(d->scale)) return GSA_ERR_INVALID_ARGUMENT;
    for (int h = 0; h < d->H; ++h) {
        if (d->head_classes[h] > 2) return GSA_ERR_INVALID_ARGUMENT;
        if (!((csr->classes >> d->head_classes[h]) & 1)) return GSA_ERR_INVALID_ARGUMENT;   // lists not built
        cls[h] = d->head_classes[h];
    }
    if (d->dtype != GSA_F32 && d->dtype != GSA_BF16) return GSA_ERR_INVALID_ARGUMENT;
    return GSA_OK;
}

}  // namespace

extern "C" {

int64_t gsa_csr_capacity(int32_t nblk) {
    if (nblk < 0) return 0;
    return static_cast<int64_t>(nblk) * (nblk + 1) / 2;
}

gsa_status gsa_block_lengths(const uint8_t* bytes, int32_t B, int64_t L, int32_t b, int32_t* lengths, void* stream) {
    const gsa::CallRange nvtx_range("gsa_block_lengths");
    if (!bytes || !lengths || B < 1 || b < 1 || b > GSA_MAX_BLOCK_BYTES || L < b || L % b != 0)
        return GSA_ERR_INVALID_ARGUMENT;
    const int64_t total = static_cast<int64_t>(B) * (L / b);
    if (b <= 32) return launch_lengths_lane<32>(bytes, b, total, lengths, as_stream(stream));
    if (b <= 64) return launch_lengths_lane<64>(bytes, b, total, lengths, as_stream(stream));
    return launch_lengths_lane<128>(bytes, b, total, lengths, as_stream(stream));
}

gsa_status gsa_literal_flags(const int32_t* lengths, int32_t B, int32_t nblk, uint8_t* flags, void* stream) {
    const gsa::CallRange nvtx_range("gsa_literal_flags");
    if (!lengths || !flags || B < 1 || nblk < 1) return GSA_ERR_INVALID_ARGUMENT;
    gsa::mask::literal_flags_kernel<<<B, 256, 0, as_stream(stream)>>>(lengths, nblk, flags);
    return launch_status();
}

gsa_status gsa_build_block_csr(const uint8_t* flags, int32_t w, const uint8_t* head_classes, int32_t H,
                               gsa_block_csr* csr, void* stream) {
    const gsa::CallRange nvtx_range("gsa_build_block_csr");
    if (!flags || !csr || w < 0) return GSA_ERR_INVALID_ARGUMENT;
    int classes = 7;
    if (head_classes) {
        if (H < 1 || H > GSA_MAX_HEADS) return GSA_ERR_INVALID_ARGUMENT;
        classes = 0;
        for (int h = 0; h < H; ++h) {
            if (head_classes[h] > 2) return GSA_ERR_INVALID_ARGUMENT;
            classes |= 1 << head_classes[h];
        }
    }
    if (csr->B < 1 || csr->nblk < 1 || !csr->row_ptr || !csr->col_idx || !csr->col_ptr || !csr->row_idx ||
        !csr->q_order || !csr->k_order)
        return GSA_ERR_INVALID_ARGUMENT;
    if (csr->nblk > gsa::mask::kMaxBlocksCsr) return GSA_ERR_UNSUPPORTED;
    if (csr->capacity < gsa_csr_capacity(csr->nblk)) return GSA_ERR_CAPACITY;
    gsa::mask::CsrArgs a;
    a.flags = flags;
    a.nblk = csr->nblk;
    a.w = w;
    a.cap = csr->capacity;
    a.row_ptr = csr->row_ptr;
    a.col_idx = csr->col_idx;
    a.col_ptr = csr->col_ptr;
    a.row_idx = csr->row_idx;
    a.q_order = csr->q_order;
    a.k_order = csr->k_order;
    int ncls = 0;
    for (int c = 0; c < 3; ++c)
        if ((classes >> c) & 1) a.cls[ncls++] = c;
    const size_t smem = gsa::mask::csr_smem_bytes(csr->nblk);
    if (!gsa::smem_opt_in(gsa::mask::build_csr_kernel,
                          static_cast<int>(gsa::mask::csr_smem_bytes(gsa::mask::kMaxBlocksCsr))))
        return GSA_ERR_CUDA;
    csr->w = w;
    csr->classes = classes;
    dim3 grid(ncls, csr->B);
    gsa::mask::build_csr_kernel<<<grid, gsa::mask::kThreads, smem, as_stream(stream)>>>(a);
    return launch_status();
}

gsa_status gsa_build_fixed_csr(int32_t kind, int32_t w, int32_t g, int32_t r, const uint32_t* rnd,
                               gsa_block_csr* csr, void* stream) {
    const gsa::CallRange nvtx_range("gsa_build_fixed_csr");
    if (!csr || (kind != GSA_FIXED_LONGFORMER && kind != GSA_FIXED_BIGBIRD) || w < 0 || g < 0 || r < 0)
        return GSA_ERR_INVALID_ARGUMENT;
    if (kind == GSA_FIXED_LONGFORMER) r = 0;
    if (r > 0 && !rnd) return GSA_ERR_INVALID_ARGUMENT;
    if (csr->B < 1 || csr->nblk < 1 || !csr->row_ptr || !csr->col_idx || !csr->col_ptr || !csr->row_idx ||
        !csr->q_order || !csr->k_order)
        return GSA_ERR_INVALID_ARGUMENT;
    if (csr->nblk > gsa::fixed::kMaxBlocks || r > gsa::fixed::kMaxRandom) return GSA_ERR_UNSUPPORTED;
    if (csr->capacity < gsa_csr_capacity(csr->nblk)) return GSA_ERR_CAPACITY;
    csr->w = w;
    csr->classes = 7;
    gsa::fixed::FixedArgs a;
    a.kind = kind;
    a.nblk = csr->nblk;
    a.w = w;
    a.g = g;
    a.r = r;
    a.rnd = rnd;
    a.cap = csr->capacity;
    a.row_ptr = csr->row_ptr;
    a.col_idx = csr->col_idx;
    a.col_ptr = csr->col_ptr;
    a.row_idx = csr->row_idx;
    a.q_order = csr->q_order;
    a.k_order = csr->k_order;
    if (!gsa::smem_opt_in(gsa::fixed::build_fixed_csr_kernel,
                          static_cast<int>(gsa::fixed::smem_bytes(gsa::fixed::kMaxBlocks, gsa::fixed::kMaxRandom))))
        return GSA_ERR_CUDA;
    dim3 grid(3, csr->B);
    gsa::fixed::build_fixed_csr_kernel<<<grid, gsa::fixed::kThreads, gsa::fixed::smem_bytes(csr->nblk, r),
                                         as_stream(stream)>>>(a);
    return launch_status();
}

gsa_status gsa_mask_pipeline(const uint8_t* bytes, int32_t B, int64_t L, int32_t b, int32_t w,
                             const uint8_t* head_classes, int32_t H, int32_t* lengths, uint8_t* flags,
                             gsa_block_csr* csr, int32_t* counter, void* stream) {
    const gsa::CallRange nvtx_range("gsa_mask_pipeline");
    if (!bytes || !lengths || !flags || !csr || !counter || B < 1 || b < 1 || b > GSA_MAX_BLOCK_BYTES ||
        L < b || L % b != 0 || w < 0)
        return GSA_ERR_INVALID_ARGUMENT;
    const int64_t nblk = L / b;
    if (csr->B != B || csr->nblk != nblk || !csr->row_ptr || !csr->col_idx || !csr->col_ptr || !csr->row_idx ||
        !csr->q_order || !csr->k_order)
        return GSA_ERR_INVALID_ARGUMENT;
    int classes = 7;
    if (head_classes) {
        if (H < 1 || H > GSA_MAX_HEADS) return GSA_ERR_INVALID_ARGUMENT;
        classes = 0;
        for (int h = 0; h < H; ++h) {
            if (head_classes[h] > 2) return GSA_ERR_INVALID_ARGUMENT;
            classes |= 1 << head_classes[h];
        }
    }
    if (nblk > GSA_MAX_PIPELINE_BLOCKS) return GSA_ERR_UNSUPPORTED;
    if (csr->capacity < gsa_csr_capacity(static_cast<int32_t>(nblk))) return GSA_ERR_CAPACITY;
    const int64_t total = static_cast<int64_t>(B) * nblk;
    gsa::pipeline::PipeArgs P{};
    P.bytes = bytes;
    P.b = b;
    P.B = B;
    P.nblk = static_cast<int>(nblk);
    P.total = total;
    P.lengths = lengths;
    P.flags = flags;
    P.counter = counter;
    for (int c = 1; c < 3; ++c)
        if ((classes >> c) & 1) P.per[P.nper++] = c;
    gsa::mask::CsrArgs& a = P.a;
    a.flags = flags;
    a.nblk = static_cast<int>(nblk);
    a.w = w;
    a.cap = csr->capacity;
    a.row_ptr = csr->row_ptr;
    a.col_idx = csr->col_idx;
    a.col_ptr = csr->col_ptr;
    a.row_idx = csr->row_idx;
    a.q_order = csr->q_order;
    a.k_order = csr->k_order;
    gsa_status st;
    if (b <= 32) st = launch_pipeline<32>(P, as_stream(stream));
    else if (b <= 64) st = launch_pipeline<64>(P, as_stream(stream));
    else st = launch_pipeline<128>(P, as_stream(stream));
    if (st != GSA_OK) return st;
    csr->w = w;
    // the local class's lists are implicit: the attention kernels derive them from (nblk, w)
    csr->classes = classes | ((classes & 1) ? 8 : 0);
    return GSA_OK;
}

gsa_status gsa_attn_fwd(const void* q, const void* k, const void* v, const gsa_block_csr* csr,
                        const gsa_attn_desc* desc, void* o, float* lse, void* stream) {
    const gsa::CallRange nvtx_range("gsa_attn_fwd");
    if (!q || !k || !v || !o) return GSA_ERR_INVALID_ARGUMENT;
    uint8_t cls[GSA_MAX_HEADS];
    gsa_status st = check_attn(desc, csr, cls);
    if (st != GSA_OK) return st;
    const float scale = desc->scale > 0.f ? desc->scale : 1.f / std::sqrt(static_cast<float>(desc->d));
    const cudaStream_t cs = as_stream(stream);

    if (desc->dtype == GSA_F32) {
        if (desc->b > 128 || !(desc->d == 16 || desc->d == 32 || desc->d == 64 || desc->d == 128) || desc->layout)
            return GSA_ERR_UNSUPPORTED;
        gsa::f32::Params p;
        p.q = static_cast<const float*>(q);
        p.k = static_cast<const float*>(k);
        p.v = static_cast<const float*>(v);
        p.o = static_cast<float*>(o);
        p.lse = lse;
        p.row_ptr = csr->row_ptr;
        p.col_idx = csr->col_idx;
        p.cap = csr->capacity;
        p.S = desc->B;
        p.H = desc->H;
        p.nblk = csr->nblk;
        p.b = desc->b;
        p.L = desc->L;
        p.scale = scale;
        std::memcpy(p.cls, cls, desc->H);
        p.local_implicit = (csr->classes >> 3) & 1;
        p.w = csr->w;
        dim3 grid(csr->nblk, desc->H, desc->B);
        const size_t smem = 3u * desc->b * desc->d * sizeof(float);
        bool opted = false;
        switch (desc->d) {
            case 16: opted = gsa::smem_opt_in(gsa::f32::attn_fwd_f32_kernel<16>, 3 * 128 * 16 * 4); break;
            case 32: opted = gsa::smem_opt_in(gsa::f32::attn_fwd_f32_kernel<32>, 3 * 128 * 32 * 4); break;
            case 64: opted = gsa::smem_opt_in(gsa::f32::attn_fwd_f32_kernel<64>, 3 * 128 * 64 * 4); break;
            default: opted = gsa::smem_opt_in(gsa::f32::attn_fwd_f32_kernel<128>, 3 * 128 * 128 * 4); break;
        }
        if (!opted) return GSA_ERR_CUDA;
        switch (desc->d) {
            case 16: gsa::f32::attn_fwd_f32_kernel<16><<<grid, 128, smem, cs>>>(p); break;
            case 32: gsa::f32::attn_fwd_f32_kernel<32><<<grid, 128, smem, cs>>>(p); break;
            case 64: gsa::f32::attn_fwd_f32_kernel<64><<<grid, 128, smem, cs>>>(p); break;
            default: gsa::f32::attn_fwd_f32_kernel<128><<<grid, 128, smem, cs>>>(p); break;
        }
        return launch_status();
    }

    // bf16 tensor-core path
    if (desc->b != gsa::bf16::kBlk || !(desc->d == 64 || desc->d == 128) || csr->nblk > GSA_MAX_BLOCKS_BF16)
        return GSA_ERR_UNSUPPORTED;
    if (!lse || !al16(q) || !al16(k) || !al16(v) || !al16(o)) return GSA_ERR_INVALID_ARGUMENT;
    const uint64_t rows = static_cast<uint64_t>(desc->B) * desc->H * desc->L;
    if (rows >= (1ull << 31)) return GSA_ERR_UNSUPPORTED;
    gsa::TokLayout lq, lo;
    st = resolve_layout(desc, &lq, &lo);
    if (st != GSA_OK) return st;
    const bool k4 = !gsa::is_dense(lq, desc->d, desc->L, desc->H);
    CUtensorMap tq, tk, tv;
    if (!gsa::make_tmap_tok(&tq, q, desc->d, desc->L, desc->H, desc->B, lq, k4) ||
        !gsa::make_tmap_tok(&tk, k, desc->d, desc->L, desc->H, desc->B, lq, k4) ||
        !gsa::make_tmap_tok(&tv, v, desc->d, desc->L, desc->H, desc->B, lq, k4))
        return GSA_ERR_CUDA;
    gsa::bf16::FwdParams p{};
    p.row_ptr = csr->row_ptr;
    p.col_idx = csr->col_idx;
    p.q_order = csr->q_order;
    p.cap = csr->capacity;
    p.S = desc->B;
    p.H = desc->H;
    p.nblk = csr->nblk;
    p.L = desc->L;
    p.o = static_cast<__nv_bfloat16*>(o);
    p.lo = lo;
    p.lse = lse;
    p.scale_log2 = scale * 1.4426950408889634f;
    std::memcpy(p.cls, cls, desc->H);
    p.local_implicit = (csr->classes >> 3) & 1;
    p.w = csr->w;
    dim3 grid(desc->B * desc->H, (csr->nblk + 1) / 2);
    if (GSA_FWD_PERSIST) {
        p.ticket = fwd_ticket_slot();
        if (!p.ticket) return GSA_ERR_CUDA;
        const int64_t items = static_cast<int64_t>(desc->B) * desc->H * ((csr->nblk + 1) / 2);
        if (desc->d == 64)
            return k4 ? launch_fwd_persist<64, true>(items, tq, tk, tv, p, cs)
                      : launch_fwd_persist<64, false>(items, tq, tk, tv, p, cs);
        return k4 ? launch_fwd_persist<128, true>(items, tq, tk, tv, p, cs)
                  : launch_fwd_persist<128, false>(items, tq, tk, tv, p, cs);
    }
    if (desc->d == 64)
        return k4 ? launch_fwd<64, true>(grid, tq, tk, tv, p, cs) : launch_fwd<64, false>(grid, tq, tk, tv, p, cs);
    return k4 ? launch_fwd<128, true>(grid, tq, tk, tv, p, cs) : launch_fwd<128, false>(grid, tq, tk, tv, p, cs);
}

size_t gsa_attn_bwd_workspace(const gsa_attn_desc* desc) {
    if (!desc || desc->B < 1 || desc->H < 1 || desc->L < 1) return 0;
    const size_t rows = static_cast<size_t>(desc->B) * desc->H * desc->L;
    return 2 * sizeof(float) * ((rows + 63) & ~size_t(63)) + 256;   // D, LSE log2(e), then work counters
}

gsa_status gsa_attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                        const gsa_block_csr* csr, const gsa_attn_desc* desc, void* dq, void* dk, void* dv,
                        void* workspace, size_t ws_bytes, void* stream) {
    const gsa::CallRange nvtx_range("gsa_attn_bwd");
    if (!q || !k || !v || !o || !lse || !dO || !dq || !dk || !dv || !workspace) return GSA_ERR_INVALID_ARGUMENT;
    uint8_t cls[GSA_MAX_HEADS];
    gsa_status st = check_attn(desc, csr, cls);
    if (st != GSA_OK) return st;
    if (ws_bytes < gsa_attn_bwd_workspace(desc)) return GSA_ERR_CAPACITY;
    if (desc->dtype != GSA_BF16) return GSA_ERR_UNSUPPORTED;
    if (desc->b != gsa::bf16::kBlk || !(desc->d == 64 || desc->d == 128) || csr->nblk > GSA_MAX_BLOCKS_BF16)
        return GSA_ERR_UNSUPPORTED;
    const uint64_t rows = static_cast<uint64_t>(desc->B) * desc->H * desc->L;
    if (rows >= (1ull << 31)) return GSA_ERR_UNSUPPORTED;
    if (!al16(q) || !al16(k) || !al16(v) || !al16(o) || !al16(dO) || !al16(dq) || !al16(dk) || !al16(dv))
        return GSA_ERR_INVALID_ARGUMENT;
    gsa::TokLayout lq, lo;
    st = resolve_layout(desc, &lq, &lo);
    if (st != GSA_OK) return st;
    const float scale = desc->scale > 0.f ? desc->scale : 1.f / std::sqrt(static_cast<float>(desc->d));
    return gsa::bwd::launch(q, k, v, o, lse, dO, csr, desc, cls, scale, dq, dk, dv, static_cast<float*>(workspace),
                            lq, lo, as_stream(stream));
}

gsa_status gsa_attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                                const void* dO, const gsa_block_csr* csr, const gsa_attn_desc* desc, void* dq,
                                void* dk, void* dv, void* stream) {
    const gsa::CallRange nvtx_range("gsa_attn_bwd_noalloc");
    if (!q || !k || !v || !o || !lse || !dO || !dq || !dk || !dv) return GSA_ERR_INVALID_ARGUMENT;
    uint8_t cls[GSA_MAX_HEADS];
    gsa_status st = check_attn(desc, csr, cls);
    if (st != GSA_OK) return st;
    if (desc->dtype != GSA_BF16) return GSA_ERR_UNSUPPORTED;
    if (desc->b != gsa::bf16::kBlk || !(desc->d == 64 || desc->d == 128) || csr->nblk > GSA_MAX_BLOCKS_BF16)
        return GSA_ERR_UNSUPPORTED;
    const int64_t rows = static_cast<int64_t>(desc->B) * desc->H * desc->L;
    if (rows > kNoAllocRows) return GSA_ERR_CAPACITY;
    float* scratch = noalloc_scratch(&st);
    if (st != GSA_OK) return st;
    const float scale = desc->scale > 0.f ? desc->scale : 1.f / std::sqrt(static_cast<float>(desc->d));
    if (!al16(q) || !al16(k) || !al16(v) || !al16(o) || !al16(dO) || !al16(dq) || !al16(dk) || !al16(dv))
        return GSA_ERR_INVALID_ARGUMENT;
    gsa::TokLayout lq, lo;
    st = resolve_layout(desc, &lq, &lo);
    if (st != GSA_OK) return st;
    return gsa::bwd::launch(q, k, v, o, lse, dO, csr, desc, cls, scale, dq, dk, dv, scratch, lq, lo,
                            as_stream(stream));
}

int64_t gsa_attn_bwd_noalloc_max_rows(void) { return kNoAllocRows; }

gsa_status gsa_device_error(int32_t* code, int32_t clear) {
    const gsa::CallRange nvtx_range("gsa_device_error");
    if (!code) return GSA_ERR_INVALID_ARGUMENT;
    if (cudaDeviceSynchronize() != cudaSuccess) return GSA_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, gsa::g_device_error, sizeof(int)) != cudaSuccess) return GSA_ERR_CUDA;
    if (clear && v != 0) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(gsa::g_device_error, &zero, sizeof(int)) != cudaSuccess) return GSA_ERR_CUDA;
    }
    *code = v;
    return v ? GSA_ERR_TIMEOUT : GSA_OK;
}

const char* gsa_status_string(gsa_status s) {
    switch (s) {
        case GSA_OK: return "ok";
        case GSA_ERR_INVALID_ARGUMENT: return "invalid argument";
        case GSA_ERR_UNSUPPORTED: return "unsupported configuration";
        case GSA_ERR_CAPACITY: return "buffer too small";
        case GSA_ERR_CUDA: return "CUDA error";
        case GSA_ERR_TIMEOUT: return "device wait timed out";
    }
    return "unknown status";
}

}  // extern "C"

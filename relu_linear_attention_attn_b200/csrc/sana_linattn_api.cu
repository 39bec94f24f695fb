// C ABI of the SANA linear-attention library: argument validation, workspace
// planning and kernel launches.  No allocation, no host synchronisation.
#include "../../include/sana_linattn.h"
#include "../../include/sana_mixffn.h"

#include <math.h>
#include <stdint.h>

#include <mutex>

#include "sana_common.cuh"
#include "simt_kernels.cuh"
#include "sm100_primitives.cuh"
#include "tc_kernels.cuh"
#include "fused_kernels.cuh"
#include "backward_tc_kernels.cuh"
#include "quant_kernels.cuh"
#include "causal_kernels.cuh"
#include "backward_kernels.cuh"
#include "mixffn_kernels.cuh"
#include "causal_tc_kernels.cuh"
#include "short_tc_kernels.cuh"

namespace sana {
namespace {

constexpr int64_t kSplitTile = 128;     // tokens per split are a multiple of this
constexpr int kTargetCtas = 4 * 148;    // pass-1 CTAs to aim for (4 per SM on 148 SMs)
constexpr int kMaxSplits = 64;

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Split-N plan for pass 1: a fixed function of (B, N, H), so results are
// reproducible bit for bit.
struct Plan {
    int S;            // splits per (b, h)
    int64_t tps;      // tokens per split
};

Plan make_plan(int64_t B, int64_t N, int H) {
    const int64_t bh = B * (int64_t)H;
    const int64_t max_by_tokens = (N + kSplitTile - 1) / kSplitTile;
    int64_t S = (kTargetCtas + bh - 1) / bh;
    if (S > max_by_tokens) S = max_by_tokens;
    if (S > kMaxSplits) S = kMaxSplits;
    if (S < 1) S = 1;
    int64_t tps = (N + S - 1) / S;
    tps = (tps + kSplitTile - 1) / kSplitTile * kSplitTile;
    S = (N + tps - 1) / tps;   // drop splits that would be empty
    if (S < 1) S = 1;
    return Plan{(int)S, tps};
}

// Plans of the persistent tensor-core passes.  The CTA count is the device's SM
// count capped at kMaxPersistentCtas; workspace sizes use the cap, which bounds
// every smaller count.
constexpr int kMaxPersistentCtas = 160;
constexpr int kP1StageTok = p1::kStageTok;
#ifndef SANA_MIN_ITEMS
#define SANA_MIN_ITEMS 4
#endif
constexpr int kMinItemsPerCta = SANA_MIN_ITEMS;

struct PersistPlan1 {
    int G, R, Smax, P;   // head groups, stages per row, partial slots per row, CTAs
    int64_t T;           // work items
};

PersistPlan1 make_plan_p1(int64_t B, int64_t N, int H, int P) {
    PersistPlan1 p{};
    p.G = (H + p1::kGroupHeads - 1) / p1::kGroupHeads;
    p.R = (int)((N + kP1StageTok - 1) / kP1StageTok);
    p.T = B * p.G * (int64_t)p.R;
    // At least kMinItemsPerCta stages per CTA (small problems use fewer SMs, and
    // a row is split among fewer partial states); never an empty range, since the
    // slot count of a row counts every CTA between the owners of its first and
    // last items.
    const int64_t cap = (p.T + kMinItemsPerCta - 1) / kMinItemsPerCta;
    p.P = (int)(cap < P ? cap : P);
    P = p.P;
    // A row's R consecutive items meet at most 1 + ceil((R-1)/L) ranges of length
    // >= L = floor(T/P), and never more than R of them.
    const int64_t L = p.T / P;
    int64_t smax = p.R;
    if (L >= 1) {
        const int64_t bound = 1 + (p.R - 1 + L - 1) / L;
        if (bound < smax) smax = bound;
    }
    p.Smax = (int)smax;
    return p;
}

struct PersistPlan2 {
    int Pp, R, P;        // head pairs, tiles per row, CTAs
    int64_t T;
};

PersistPlan2 make_plan_p2(int64_t B, int64_t N, int H, int P) {
    PersistPlan2 p{};
    p.Pp = (H + p2::kPairHeads - 1) / p2::kPairHeads;
    p.R = (int)((N + p2::kTileTok - 1) / p2::kTileTok);
    p.T = B * p.Pp * (int64_t)p.R;
    p.P = (int)(p.T < P ? p.T : P);
    return p;
}

// Plan of the fused kernels: CTA (s, g, b) takes tiles [s*tps, (s+1)*tps) of batch
// b for head group g; about one wave of one CTA per SM.
struct FusedPlan {
    int G, tiles, S, tps;
};

FusedPlan make_plan_fused(int64_t B, int64_t N, int H, int P) {
    FusedPlan f{};
    f.G = (H + fz::kGroupHeads - 1) / fz::kGroupHeads;
    f.tiles = (int)((N + fz::kTileTok - 1) / fz::kTileTok);
    int64_t S = P / (B * f.G);
    if (S < 1) S = 1;
    if (S > f.tiles) S = f.tiles;
    f.tps = (int)((f.tiles + S - 1) / S);
    f.S = (f.tiles + f.tps - 1) / f.tps;
    return f;
}

int max_splits(int64_t B, int64_t N, int H) {
    const int a = make_plan(B, N, H).S, b = make_plan_p1(B, N, H, kMaxPersistentCtas).Smax;
    return a > b ? a : b;
}

// Workspace layout of the unfused path: [partials B*H*S*1056 fp32][state B*H*1056 fp32].
struct WsLayout {
    size_t part_off, kv_off, counters_off, total;
};

WsLayout ws_layout(int64_t B, int64_t N, int C, int H, bool fused) {
    const int S = fused ? make_plan_fused(B, N, H, kMaxPersistentCtas).S : max_splits(B, N, H);
    WsLayout w{};
    size_t off = 0;
    w.counters_off = off;
    off = align_up(off + (size_t)B * ((H + 3) / 4) * sizeof(int), 256);
    w.part_off = off;
    off = align_up(off + (size_t)B * H * S * kStateFloats * sizeof(float), 256);
    w.kv_off = off;
    off = align_up(off + (size_t)B * H * kStateFloats * sizeof(float), 256);
    w.total = off;
    return w;
}

bool aligned(const void* p, uintptr_t a) { return ((uintptr_t)p & (a - 1)) == 0; }

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
    if (!a || !b || na == 0 || nb == 0) return false;
    const uintptr_t a0 = (uintptr_t)a, b0 = (uintptr_t)b;
    return a0 < b0 + nb && b0 < a0 + na;
}

int check_dims(int64_t B, int64_t N, int C, int H) {
    if (B < 0 || N < 0 || C <= 0 || H <= 0 || C % H != 0) return SANA_EINVAL;
    if (C / H != kD) return SANA_EUNSUPPORTED;
    if (B > 65535 || H > 65535) return SANA_EUNSUPPORTED;     // grid z / y limits
    if (N > ((int64_t)1 << 40) || B * N > ((int64_t)1 << 40)) return SANA_EUNSUPPORTED;
    return SANA_OK;
}

int check_eps(float eps) { return (eps >= 0.f && isfinite(eps)) ? SANA_OK : SANA_EINVAL; }

int check_gains(const float* gq, const float* gk) {
    if ((gq == nullptr) != (gk == nullptr)) return SANA_EINVAL;
    if (gq && (!aligned(gq, 4) || !aligned(gk, 4))) return SANA_EALIGN;
    return SANA_OK;
}

size_t elem_size(sana_dtype dt) { return dt == SANA_BF16 ? 2 : 4; }

int launch_status() {
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? SANA_OK : SANA_ECUDA;
}

// Pass 1 + combine on inputs of element type T with row strides ldk, ldv.
template <typename T>
void launch_state(const T* k, const T* v, const float* gk, float* part, float* kv,
                  int64_t B, int64_t N, int H, int64_t ldk, int64_t ldv, float eps,
                  const Plan& p, cudaStream_t st) {
    const dim3 g1(p.S, H, (unsigned)B);
    kv_partial_simt<T><<<g1, 128, 0, st>>>(k, v, gk, part, N, H, ldk, ldv, p.S, p.tps, eps,
                                           gk != nullptr);
    kv_combine<<<(unsigned)(B * H), 256, 0, st>>>(part, kv, p.S);
}

template <typename TI, typename TO>
void launch_apply(const TI* q, const float* gq, const float* kv, TO* out, int64_t B, int64_t N,
                  int H, int64_t ldq, int64_t ldo, float eps, cudaStream_t st) {
    const dim3 g((unsigned)((N + 127) / 128), H, (unsigned)B);
    apply_simt<TI, TO><<<g, 128, 0, st>>>(q, gq, kv, out, N, H, ldq, ldo, eps, gq != nullptr);
}

// ---------------------------------------------------------------- TMA tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            fn = (EncodeTiledFn)p;
    }
    return fn;
}

// A (B, N, C) bf16 (or int8) tensor seen by TMA as 3-D (C, N, B), boxes of 128
// bytes of channels (64 bf16 or 128 int8) x `rows` tokens x 1 batch, 128-byte
// swizzle.  Rows past N read as zeros and are not written by stores, so a tile
// never crosses into the next batch item.
bool make_tmap_bnc(CUtensorMap* m, const void* base, int64_t B, int64_t N, int C, int rows,
                   bool i8 = false) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t es = i8 ? 1 : 2;
    const cuuint64_t dims[3] = {(cuuint64_t)C, (cuuint64_t)N, (cuuint64_t)B};
    const cuuint64_t strides[2] = {(cuuint64_t)C * es, (cuuint64_t)N * C * es};
    const cuuint32_t box[3] = {i8 ? 128u : 64u, (cuuint32_t)rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, i8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
              const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Wqkv (C, 3C) row-major seen by TMA as 3-D (n within a section, section, k) =
// (C, 3, C): boxes of 128 bytes of n (64 bf16 or 128 int8) x 1 section x as many
// k, 128-byte swizzle.  Columns past a section's C read as zeros, so head groups
// past H never pick up the next section.  (Bytes are moved as unsigned 8-bit; the
// UMMA reads them as signed int8.)
bool make_tmap_w(CUtensorMap* m, const void* W, int C, bool i8 = false) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t es = i8 ? 1 : 2;
    const cuuint64_t dims[3] = {(cuuint64_t)C, 3, (cuuint64_t)C};
    const cuuint64_t strides[2] = {(cuuint64_t)C * es, (cuuint64_t)C * 3 * es};
    const cuuint32_t box[3] = {i8 ? 128u : 64u, 1, i8 ? 128u : 64u};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, i8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
              const_cast<void*>(W), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The tensor-core kernels keep the gains of every channel in shared memory, so they
// take C <= 4096 (H <= 128); wider problems run the CUDA-core kernels.
bool tc_path(sana_dtype dt, int C) { return dt == SANA_BF16 && C <= p1::kGainCache; }

// Per-device setup of the persistent kernels: dynamic shared memory opt-in and
// the CTA count (SM count, capped).  Returns 0 on failure.
int persistent_ctas() {
    static int ctas[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    if (ctas[dev]) return ctas[dev];
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        sms <= 0)
        return 0;
    if (cudaFuncSetAttribute(kv_partials_persistent<false>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, p1::kSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(kv_partials_persistent<true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, p1::kSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(kv_partials_persistent<false, true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, p1::kSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(apply_persistent, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             p2::kSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(fused_kv<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             f1::kSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(fused_qo<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             f2::kSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(fused_kv<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             f1::kSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(fused_qo<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             f2::kSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(causal_apply_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             ca::kSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(bwd_key_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             bk::kSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(bwd_query_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             bq::kSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(forward_short_cluster, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             sc::kSmemBytes) != cudaSuccess)
        return 0;
    // each persistent kernel must fit one CTA on an SM (registers, threads, smem)
    int n1 = 0, n2 = 0, n3 = 0, n4 = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n1, kv_partials_persistent<false>,
                                                      p1::kThreads, p1::kSmemBytes) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n2, apply_persistent, p2::kThreads,
                                                      p2::kSmemBytes) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n3, fused_kv<false>, f1::kThreads,
                                                      f1::kSmemBytes) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n4, fused_qo<false>, f2::kThreads,
                                                      f2::kSmemBytes) != cudaSuccess ||
        n1 < 1 || n2 < 1 || n3 < 1 || n4 < 1)
        return 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n3, fused_kv<true>, f1::kThreads,
                                                      f1::kSmemBytes) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n4, fused_qo<true>, f2::kThreads,
                                                      f2::kSmemBytes) != cudaSuccess ||
        n3 < 1 || n4 < 1)
        return 0;
    ctas[dev] = sms < kMaxPersistentCtas ? sms : kMaxPersistentCtas;
    return ctas[dev];
}

// Launch with programmatic stream serialization: the kernel may start while the
// previous grid in the stream finishes, and waits for it (griddepcontrol.wait)
// before it touches global memory.
template <typename... Args>
int launch_pdl(void (*kernel)(Args...), dim3 grid, int threads, int smem, cudaStream_t st,
               bool pdl, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, args...) == cudaSuccess ? SANA_OK : SANA_ECUDA;
}

// bf16 pass 1 on the tensor cores: per-row-segment partial states into `part`
// ([B][H][Smax][D+1][D]); nothing else is written.
int launch_partials_tc(const void* k, const void* v, const float* gk, float* part, int64_t B,
                       int64_t N, int C, int H, float eps, cudaStream_t st,
                       PersistPlan1* plan_out, const float* w = nullptr) {
    const int P = persistent_ctas();
    if (P == 0) return SANA_ECUDA;
    CUtensorMap tk, tv;
    if (!make_tmap_bnc(&tk, k, B, N, C, kP1StageTok) ||
        !make_tmap_bnc(&tv, v, B, N, C, kP1StageTok))
        return SANA_ECUDA;
    const PersistPlan1 pl = make_plan_p1(B, N, H, P);
    P1Args a{};
    a.gk = gk; a.part = part; a.T = pl.T; a.Cc = 1;
    a.N = (int)N; a.H = H; a.G = pl.G; a.R = pl.R; a.Smax = pl.Smax; a.P = pl.P;
    a.eps = eps; a.norm = gk != nullptr; a.w = w;
    if (plan_out) *plan_out = pl;
    if (w)
        return launch_pdl(kv_partials_persistent<false, true>, dim3(pl.P), p1::kThreads,
                          p1::kSmemBytes, st, true, tk, tv, a);
    return launch_pdl(kv_partials_persistent<false>, dim3(pl.P), p1::kThreads, p1::kSmemBytes, st,
                      true, tk, tv, a);
}

// The final states kv [B][H][D][D+1] from pass-1 partials (right behind pass 1).
int launch_combine_tc(const float* part, float* kv, int64_t B, int H, const PersistPlan1& pl,
                      cudaStream_t st) {
    return launch_pdl(kv_combine_partials, dim3((unsigned)(B * H)), 256, 0, st, true,
                      (const float*)part, kv, H, pl.G, (int64_t)pl.R, pl.T, (int64_t)pl.P,
                      pl.Smax);
}

// bf16 pass 2 on the tensor cores.  With kv == nullptr it sums the pass-1 partials
// of plan p1 itself and is launched right behind pass 1 (its Q stream starts while
// pass 1 finishes; only the partial reads wait for pass 1).
int launch_apply_tc(const void* q, const float* gq, const float* kv, const float* part,
                    const PersistPlan1* p1pl, void* out, int64_t B, int64_t N, int C, int H,
                    float eps, cudaStream_t st) {
    const int P = persistent_ctas();
    if (P == 0) return SANA_ECUDA;
    CUtensorMap tq, to;
    if (!make_tmap_bnc(&tq, q, B, N, C, p2::kTileTok) ||
        !make_tmap_bnc(&to, out, B, N, C, p2::kTileTok))
        return SANA_ECUDA;
    const PersistPlan2 pl = make_plan_p2(B, N, H, P);
    P2Args a{};
    a.kv = kv; a.part = part; a.gq = gq; a.T = pl.T; a.N = (int)N; a.H = H; a.Pp = pl.Pp;
    a.R = pl.R; a.P = pl.P; a.eps = eps; a.norm = gq != nullptr;
    if (kv == nullptr) {
        if (!p1pl || !part) return SANA_EINVAL;
        a.T1 = p1pl->T; a.P1 = p1pl->P; a.R1 = p1pl->R; a.G1 = p1pl->G; a.Smax1 = p1pl->Smax;
    }
    return launch_pdl(apply_persistent, dim3(pl.P), p2::kThreads, p2::kSmemBytes, st,
                      kv == nullptr, tq, to, a);
}

// Short sequences (bf16, N <= 128 * 8): the whole forward as one launch of
// clusters of S = ceil(N / 128) CTAs, one cluster per (b, group of 4 heads).
constexpr int64_t kShortMaxN = (int64_t)sc::kTok * sc::kMaxCluster;
// Beyond this many CTAs (about 2.7 per SM) the persistent passes, which stream
// tiles through deep rings, are faster than one tile per CTA (measured on B200 at
// N = 777 and 1024: B = 3 and below favour the clusters, B = 4 and above the passes).
constexpr int64_t kShortMaxCtas = 400;

bool short_path(int64_t B, int64_t N, int H) {
    const int64_t S = (N + sc::kTok - 1) / sc::kTok, G = (H + sc::kHeads - 1) / sc::kHeads;
    return N <= kShortMaxN && B <= 65535 && B * G * S <= kShortMaxCtas;
}

int launch_short_tc(const void* q, const void* k, const void* v, const float* gq,
                    const float* gk, void* out, int64_t B, int64_t N, int C, int H, float eps,
                    cudaStream_t st) {
    if (persistent_ctas() == 0) return SANA_ECUDA;           // the kernel attributes
    const int S = (int)((N + sc::kTok - 1) / sc::kTok);
    const int G = (H + sc::kHeads - 1) / sc::kHeads;
    CUtensorMap tq, tk, tv, to;
    if (!make_tmap_bnc(&tq, q, B, N, C, sc::kTok) || !make_tmap_bnc(&to, out, B, N, C, sc::kTok) ||
        !make_tmap_bnc(&tk, k, B, N, C, sc::kStageTok) ||
        !make_tmap_bnc(&tv, v, B, N, C, sc::kStageTok))
        return SANA_ECUDA;
    ScArgs a{};
    a.gq = gq; a.gk = gk; a.N = (int)N; a.H = H; a.S = S; a.eps = eps;
    a.norm = gq != nullptr && gk != nullptr;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)S, (unsigned)G, (unsigned)B);
    cfg.blockDim = dim3(sc::kThreads);
    cfg.dynamicSmemBytes = sc::kSmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)S;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, forward_short_cluster, tq, tk, tv, to, a) == cudaSuccess
               ? SANA_OK
               : SANA_ECUDA;
}

// The prefix (causal) form on the tensor cores (bf16): pass 1 with one row per
// 128-token chunk (the chunks' partial states), the exclusive prefix over chunks,
// then the chunked apply.  Workspace: [partials B*H*Cc*2 states][prefix B*H*Cc].
int launch_causal_tc(const void* q, const void* k, const void* v, const float* gq,
                     const float* gk, void* out, int64_t B, int64_t N, int C, int H, float eps,
                     void* workspace, cudaStream_t st) {
    const int P = persistent_ctas();
    if (P == 0) return SANA_ECUDA;
    const int64_t Cc = (N + kCausalTcChunk - 1) / kCausalTcChunk;
    constexpr int kR = kCausalTcChunk / p1::kStageTok;      // pass-1 stages per chunk
    const int G = (H + p1::kGroupHeads - 1) / p1::kGroupHeads;
    const int64_t T1 = B * G * Cc * kR;
    if (B * (int64_t)H * Cc > 0x7fffffffLL || T1 > ((int64_t)1 << 40)) return SANA_EUNSUPPORTED;
    const int64_t cap = (T1 + kMinItemsPerCta - 1) / kMinItemsPerCta;
    const int P1 = (int)(cap < P ? cap : P);
    float* part = (float*)workspace;
    float* pre = (float*)((char*)workspace +
                          align_up((size_t)B * H * Cc * 2 * kStateFloats * sizeof(float), 256));
    CUtensorMap tk, tv;
    if (!make_tmap_bnc(&tk, k, B, N, C, kP1StageTok) || !make_tmap_bnc(&tv, v, B, N, C, kP1StageTok))
        return SANA_ECUDA;
    P1Args a1{};
    a1.gk = gk; a1.part = part; a1.T = T1; a1.N = (int)N; a1.H = H; a1.G = G; a1.R = kR;
    a1.Smax = 2; a1.P = P1; a1.eps = eps; a1.norm = gk != nullptr; a1.Cc = (int)Cc;
    int rc = launch_pdl(kv_partials_persistent<true>, dim3(P1), p1::kThreads, p1::kSmemBytes, st,
                        false, tk, tv, a1);
    if (rc != SANA_OK) return rc;
    PrefixArgs ap{};
    ap.part = part; ap.pre = pre; ap.H = H; ap.G = G; ap.Cc = (int)Cc; ap.Smax = 2;
    ap.R1 = kR; ap.T1 = T1; ap.P1 = P1;
    causal_prefix_states<<<(unsigned)(B * H), kPrefixThreads, 0, st>>>(ap);
    rc = launch_status();
    if (rc != SANA_OK) return rc;
    CUtensorMap tq, tk2, tv2, to;
    if (!make_tmap_bnc(&tq, q, B, N, C, ca::kTok) || !make_tmap_bnc(&tk2, k, B, N, C, ca::kTok) ||
        !make_tmap_bnc(&tv2, v, B, N, C, ca::kTok) || !make_tmap_bnc(&to, out, B, N, C, ca::kTok))
        return SANA_ECUDA;
    CaArgs a3{};
    a3.pre = pre; a3.gq = gq; a3.gk = gk; a3.N = (int)N; a3.H = H;
    a3.Pp = (H + 1) / 2; a3.Cc = (int)Cc; a3.T = B * a3.Pp * Cc;
    a3.P = (int)(a3.T < P ? a3.T : P); a3.eps = eps; a3.norm = gq != nullptr;
    return launch_pdl(causal_apply_tc, dim3(a3.P), ca::kThreads, ca::kSmemBytes, st, true, tq, tk2, tv2,
                      to, a3);
}

// The fused variant: F1 (K, V projection + state), then F2 (Q projection + apply)
// as a programmatic dependent launch.
template <bool kI8>
int launch_fused(const void* x, const void* W, const float* sx, const float* sw, const float* gq,
                 const float* gk, void* out, int* counters, float* part, float* kv, int64_t B,
                 int64_t N, int C, int H, float eps, cudaStream_t st) {
    const int P = persistent_ctas();
    if (P == 0) return SANA_ECUDA;
    CUtensorMap tx, tw, to;
    if (!make_tmap_bnc(&tx, x, B, N, C, fz::kTileTok, kI8) || !make_tmap_w(&tw, W, C, kI8) ||
        !make_tmap_bnc(&to, out, B, N, C, fz::kTileTok))
        return SANA_ECUDA;
    const FusedPlan pl = make_plan_fused(B, N, H, P);
    if (cudaMemsetAsync(counters, 0, (size_t)B * pl.G * sizeof(int), st) != cudaSuccess)
        return SANA_ECUDA;
    F1Args a1{};
    a1.sx = sx; a1.sw = sw;
    a1.gk = gk; a1.part = part; a1.kv = kv; a1.counters = counters;
    a1.N = (int)N; a1.H = H; a1.C = C; a1.S = pl.S; a1.tps = pl.tps; a1.eps = eps;
    a1.norm = gk != nullptr;
    const dim3 grid(pl.S, pl.G, (unsigned)B);
    fused_kv<kI8><<<grid, f1::kThreads, f1::kSmemBytes, st>>>(tx, tw, a1);
    F2Args a2{};
    a2.sx = sx; a2.sw = sw;
    a2.kv = kv; a2.gq = gq; a2.N = (int)N; a2.H = H; a2.C = C; a2.tps = pl.tps; a2.eps = eps;
    a2.norm = gq != nullptr;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(f2::kThreads);   // fused_qo
    cfg.dynamicSmemBytes = f2::kSmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, fused_qo<kI8>, tx, tw, to, a2) != cudaSuccess) return SANA_ECUDA;
    return SANA_OK;
}

int validate_qkv(const void* q, const void* k, const void* v, const void* out, int64_t B,
                 int64_t N, int C, sana_dtype dtype) {
    if (dtype != SANA_BF16 && dtype != SANA_F32) return SANA_EINVAL;
    if (!q || !k || !v || !out) return SANA_EINVAL;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16))
        return SANA_EALIGN;
    const size_t bytes = (size_t)B * N * C * elem_size(dtype);
    if (overlaps(out, bytes, q, bytes) || overlaps(out, bytes, k, bytes) ||
        overlaps(out, bytes, v, bytes))
        return SANA_EINVAL;
    return SANA_OK;
}

int validate_ws(void* ws, size_t ws_bytes, size_t need) {
    if (need == 0) return SANA_OK;
    if (!ws || ws_bytes < need) return SANA_EWORKSPACE;
    if (!aligned(ws, 256)) return SANA_EALIGN;
    return SANA_OK;
}

}  // namespace

// ---------------------------------------------------------------- static scratch
// Scratch for sana_linattn_forward_noalloc: a fixed array in the module's device
// memory, created when the library's module is loaded on a device and held by
// every device that loads it until the process exits.
constexpr size_t kNoAllocScratchBytes = (size_t)16 << 20;   // 16 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[64] = {};

// Device address of g_noalloc_scratch on the current device.  In host code the
// array's name only stands in for the symbol; its device address has to be
// looked up once per device, with that device current.
int noalloc_scratch(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return SANA_ECUDA;
    if (dev < 0 || dev >= 64) return SANA_EUNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
            return SANA_ECUDA;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return SANA_OK;
}
// Target of the launch-failure self-test; never runs.
__global__ void launch_failure_selftest() {}

}  // namespace
}  // namespace sana

using namespace sana;

extern "C" {

size_t sana_linattn_workspace_bytes(int64_t B, int64_t N, int C, int H, int fused) {
    if (check_dims(B, N, C, H) != SANA_OK || B == 0 || N == 0) return 0;
    if (fused == 2) {        // the prefix form: states per chunk of every (b, h)
        // CUDA-core path: one state per 64-token chunk; tensor-core path: up to two
        // partial slots and the prefix per 128-token chunk
        const int64_t S = (N + kCausalChunk - 1) / kCausalChunk;
        const size_t simt = align_up((size_t)B * H * S * kStateFloats * sizeof(float), 256);
        const int64_t Cc = (N + kCausalTcChunk - 1) / kCausalTcChunk;
        const size_t tc = 2 * align_up((size_t)B * H * Cc * 2 * kStateFloats * sizeof(float), 256);
        return simt > tc ? simt : tc;
    }
    return ws_layout(B, N, C, H, fused != 0).total;
}

size_t sana_linattn_backward_workspace_bytes(int64_t B, int64_t N, int C, int H) {
    if (check_dims(B, N, C, H) != SANA_OK || B == 0 || N == 0) return 0;
    const int64_t tiles = (N + kBwdTile - 1) / kBwdTile;
    size_t off = 0;
    // split partials: the forward state's (either plan), then dS, dz's
    off = align_up(off + (size_t)B * H * max_splits(B, N, H) * kStateFloats * 4, 256);
    off = align_up(off + (size_t)B * H * kStateFloats * 4, 256);         // forward states
    off = align_up(off + (size_t)B * H * kStateFloats * 4, 256);         // [dS | dz]
    off = align_up(off + (size_t)B * N * H * kGrow * 4, 256);            // [dnum | dden] rows
    off = align_up(off + (size_t)2 * B * tiles * C * 4, 256);            // gain partials
    // the key side on the tensor cores: gain partials per (tile, quadrant, head pair)
    const int64_t Tk = B * ((H + 1) / 2) * tiles;
    off = align_up(off + (size_t)Tk * 4 * 2 * kD * 4, 256);
    off = align_up(off + (size_t)((H + 1) / 2) * kGainSlices * 2 * kD * 4, 256);   // their slices
    off = align_up(off + (size_t)Tk * 4 * 2 * kD * 4, 256);                         // query side
    return off;
}

// The key side of the backward on the tensor cores (bwd_key_tc): dK, dV and the
// per-tile gain partials from [dS | dz].
int launch_bwd_key_tc(const void* k, const void* v, const float* gk, const float* dsz, void* dk,
                      void* dv, float* gpart, int64_t B, int64_t N, int C, int H, float eps,
                      cudaStream_t st) {
    const int P = persistent_ctas();
    if (P == 0) return SANA_ECUDA;
    CUtensorMap tk, tv, tdk, tdv;
    if (!make_tmap_bnc(&tk, k, B, N, C, bk::kTileTok) || !make_tmap_bnc(&tv, v, B, N, C, bk::kTileTok) ||
        !make_tmap_bnc(&tdk, dk, B, N, C, bk::kTileTok) ||
        !make_tmap_bnc(&tdv, dv, B, N, C, bk::kTileTok))
        return SANA_ECUDA;
    BkArgs a{};
    a.dsz = dsz; a.gk = gk; a.k = (const bf16*)k; a.gpart = gpart;
    a.N = (int)N; a.H = H; a.Pp = (H + 1) / 2; a.R = (int)((N + bk::kTileTok - 1) / bk::kTileTok);
    a.T = B * a.Pp * (int64_t)a.R;
    a.P = (int)(a.T < P ? a.T : P);
    a.eps = eps; a.norm = gk != nullptr;
    return launch_pdl(bwd_key_tc, dim3(a.P), bk::kThreads, bk::kSmemBytes, st, true, tk, tv, tdk,
                      tdv, a);
}

// The query side of the backward on the tensor cores (bwd_query_tc): dQ, dnum (bf16,
// (B, N, C)), dden ((B, H, N) fp32) and the per-tile gain partials from the states S.
int launch_bwd_query_tc(const void* q, const void* dout, const float* gq, const float* s, void* dq,
                        void* dnum, float* dden, float* gpart, int64_t B, int64_t N, int C, int H,
                        float eps, cudaStream_t st) {
    const int P = persistent_ctas();
    if (P == 0) return SANA_ECUDA;
    CUtensorMap tq, tg, tdq, tdn;
    if (!make_tmap_bnc(&tq, q, B, N, C, bq::kTileTok) ||
        !make_tmap_bnc(&tg, dout, B, N, C, bq::kTileTok) ||
        !make_tmap_bnc(&tdq, dq, B, N, C, bq::kTileTok) ||
        !make_tmap_bnc(&tdn, dnum, B, N, C, bq::kTileTok))
        return SANA_ECUDA;
    BqArgs a{};
    a.s = s; a.gq = gq; a.q = (const bf16*)q; a.dden = dden; a.gpart = gpart;
    a.N = (int)N; a.H = H; a.Pp = (H + 1) / 2; a.R = (int)((N + bq::kTileTok - 1) / bq::kTileTok);
    a.T = B * a.Pp * (int64_t)a.R;
    a.P = (int)(a.T < P ? a.T : P);
    a.eps = eps; a.norm = gq != nullptr;
    return launch_pdl(bwd_query_tc, dim3(a.P), bq::kThreads, bq::kSmemBytes, st, true, tq, tg, tdq,
                      tdn, a);
}

// The backward forms [dS | dz] on the tensor cores (bf16 phi(Q) and dnum) from this
// many tokens on.  For very short sequences the key gradients are a small difference
// of O(1) terms (one token: dphi(K) = phi(Q) (dnum . V + dden) = O(eps)), which the
// bf16 rounding of the operands would dominate; there the fp32 CUDA-core reduction
// runs instead.  The tensor-core backward also wants 16-byte aligned gains (its
// kernels read them from global memory as 16-byte vectors); others take the CUDA-core
// path.
constexpr int64_t kBwdTcMinTokens = 128;

}  // extern "C"

namespace sana {
namespace {

// The backward; `state` is the forward's (B, H, D, D+1) state when the caller has
// it (sana_linattn_backward_with_state), else nullptr and it is formed here exactly
// as sana_linattn_kv_state forms it.
int backward_impl(const void* q, const void* k, const void* v, const float* gq,
                  const float* gk, const void* dout, void* dq, void* dk, void* dv,
                  float* dgq, float* dgk, int64_t B, int64_t N, int C, int H, float eps,
                  sana_dtype dtype, void* workspace, size_t ws_bytes, cudaStream_t stream,
                  const float* state) {
    int rc;
    if ((rc = check_dims(B, N, C, H)) != SANA_OK) return rc;
    if ((rc = check_eps(eps)) != SANA_OK) return rc;
    if ((rc = check_gains(gq, gk)) != SANA_OK) return rc;
    if (dtype != SANA_BF16 && dtype != SANA_F32) return SANA_EINVAL;
    const bool norm = gq != nullptr;
    if (norm != (dgq != nullptr) || norm != (dgk != nullptr)) return SANA_EINVAL;
    if (norm && (!aligned(dgq, 4) || !aligned(dgk, 4))) return SANA_EALIGN;
    if (B == 0 || N == 0) {
        if (norm && (cudaMemsetAsync(dgq, 0, (size_t)C * 4, stream) != cudaSuccess ||
                     cudaMemsetAsync(dgk, 0, (size_t)C * 4, stream) != cudaSuccess))
            return SANA_ECUDA;
        return SANA_OK;
    }
    if (!q || !k || !v || !dout || !dq || !dk || !dv) return SANA_EINVAL;
    const void* ins[4] = {q, k, v, dout};
    void* outs[3] = {dq, dk, dv};
    for (const void* p : ins) if (!aligned(p, 16)) return SANA_EALIGN;
    for (void* p : outs) if (!aligned(p, 16)) return SANA_EALIGN;
    const size_t bytes = (size_t)B * N * C * elem_size(dtype);
    for (void* o : outs) {
        for (const void* i : ins) if (overlaps(o, bytes, i, bytes)) return SANA_EINVAL;
        for (void* o2 : outs) if (o2 != o && overlaps(o, bytes, o2, bytes)) return SANA_EINVAL;
    }
    const size_t need = sana_linattn_backward_workspace_bytes(B, N, C, H);
    if ((rc = validate_ws(workspace, ws_bytes, need)) != SANA_OK) return rc;
    for (const void* i : ins) if (overlaps(workspace, need, i, bytes)) return SANA_EINVAL;
    for (void* o : outs) if (overlaps(workspace, need, o, bytes)) return SANA_EINVAL;
    const size_t state_bytes = (size_t)B * H * kStateFloats * sizeof(float);
    if (state) {
        if (!aligned(state, 16)) return SANA_EALIGN;
        if (overlaps(workspace, need, state, state_bytes)) return SANA_EINVAL;
        for (void* o : outs) if (overlaps(o, bytes, state, state_bytes)) return SANA_EINVAL;
    }
    const Plan p = make_plan(B, N, H);
    const int64_t tiles = (N + kBwdTile - 1) / kBwdTile;
    char* w = (char*)workspace;
    size_t off = 0;
    float* part = (float*)(w + off);
    off = align_up(off + (size_t)B * H * max_splits(B, N, H) * kStateFloats * 4, 256);
    float* Sz_ws = (float*)(w + off);
    const float* Sz = state ? state : Sz_ws;
    off = align_up(off + (size_t)B * H * kStateFloats * 4, 256);
    float* dSz = (float*)(w + off);
    off = align_up(off + (size_t)B * H * kStateFloats * 4, 256);
    float* G = (float*)(w + off);
    off = align_up(off + (size_t)B * N * H * kGrow * 4, 256);
    float* gpq = (float*)(w + off);
    float* gpk = gpq + (size_t)B * tiles * C;
    off = align_up(off + (size_t)2 * B * tiles * C * 4, 256);
    float* gpk_tc = (float*)(w + off);
    off = align_up(off + (size_t)B * ((H + 1) / 2) * tiles * 4 * 2 * kD * 4, 256);
    float* gslices = (float*)(w + off);
    off = align_up(off + (size_t)((H + 1) / 2) * kGainSlices * 2 * kD * 4, 256);
    float* gpq_tc = (float*)(w + off);
    const dim3 gs(p.S, H, (unsigned)B), gt((unsigned)tiles, H, (unsigned)B);
    const int nrm = norm ? 1 : 0;
    if (dtype == SANA_BF16) {
        // the forward state as sana_linattn_kv_state forms it (tensor-core pass 1 +
        // combine), unless the caller passed it in
        if (state) {
        } else if (tc_path(dtype, C)) {
            PersistPlan1 pl{};
            if ((rc = launch_partials_tc(k, v, gk, part, B, N, C, H, eps, stream, &pl)) != SANA_OK ||
                (rc = launch_combine_tc(part, Sz_ws, B, H, pl, stream)) != SANA_OK)
                return rc;
        } else {
            launch_state<bf16>((const bf16*)k, (const bf16*)v, gk, part, Sz_ws, B, N, H, C, C, eps,
                               p, stream);
        }
        if (tc_path(dtype, C) && N >= kBwdTcMinTokens &&
            (!norm || (aligned(gq, 16) && aligned(gk, 16)))) {
            // Query side on the tensor cores: dQ, dnum (bf16, (B, N, C)) and dden (fp32,
            // (B, H, N)) in the space of the [dnum | dden] rows (B N H (64 + 4) bytes + 16
            // of padding <= B N H 132).  Then [dS | dz] = sum_t phi(Q)_t^T [dnum_t | dden_t]
            // by pass 1 with q in K's place (its gains gq), dnum in V's and the normaliser
            // column weighted by dden; then the key side, and the gain partials' sums.
            bf16* dnum = (bf16*)G;
            float* dden = (float*)((char*)G + align_up((size_t)B * N * C * sizeof(bf16), 16));
            PersistPlan1 pl{};
            if ((rc = launch_status()) != SANA_OK ||
                (rc = launch_bwd_query_tc(q, dout, gq, Sz, dq, dnum, dden, gpq_tc, B, N, C, H, eps,
                                          stream)) != SANA_OK ||
                (rc = launch_partials_tc(q, dnum, gq, part, B, N, C, H, eps, stream, &pl, dden)) !=
                    SANA_OK ||
                (rc = launch_combine_tc(part, dSz, B, H, pl, stream)) != SANA_OK ||
                (rc = launch_bwd_key_tc(k, v, gk, dSz, dk, dv, gpk_tc, B, N, C, H, eps, stream)) !=
                    SANA_OK)
                return rc;
            if (norm) {
                const int Pp = (H + 1) / 2;
                const float* gp[2] = {gpq_tc, gpk_tc};
                float* dg[2] = {dgq, dgk};
                for (int x = 0; x < 2; ++x) {
                    gain_combine_tiles<<<dim3((unsigned)Pp, kGainSlices), 256, 0, stream>>>(
                        gp[x], gslices, (int)B, Pp, (int)tiles);
                    gain_combine_slices<<<(C + 255) / 256, 256, 0, stream>>>(gslices, dg[x], Pp, H);
                }
            }
            return launch_status();
        } else {
            bwd_query_simt<bf16><<<gt, kBwdTile, 0, stream>>>((const bf16*)q, (const bf16*)dout, gq,
                                                              Sz, (bf16*)dq, G, gpq, N, H, eps, nrm);
            outer_partial_simt<bf16><<<gs, 128, 0, stream>>>((const bf16*)q, gq, G, part, N, H,
                                                             p.S, p.tps, eps, nrm);
            kv_combine<<<(unsigned)(B * H), 256, 0, stream>>>(part, dSz, p.S);
        }
        bwd_key_simt<bf16><<<gt, kBwdTile, 0, stream>>>((const bf16*)k, (const bf16*)v, gk, dSz,
                                                        (bf16*)dk, (bf16*)dv, gpk, N, H, eps, nrm);
    } else {
        if (!state)
            launch_state<float>((const float*)k, (const float*)v, gk, part, Sz_ws, B, N, H, C, C,
                                eps, p, stream);
        bwd_query_simt<float><<<gt, kBwdTile, 0, stream>>>((const float*)q, (const float*)dout, gq,
                                                           Sz, (float*)dq, G, gpq, N, H, eps, nrm);
        outer_partial_simt<float><<<gs, 128, 0, stream>>>((const float*)q, gq, G, part, N, H, p.S,
                                                          p.tps, eps, nrm);
        kv_combine<<<(unsigned)(B * H), 256, 0, stream>>>(part, dSz, p.S);
        bwd_key_simt<float><<<gt, kBwdTile, 0, stream>>>((const float*)k, (const float*)v, gk, dSz,
                                                         (float*)dk, (float*)dv, gpk, N, H, eps,
                                                         nrm);
    }
    if (norm) {
        gain_combine<<<(C + 255) / 256, 256, 0, stream>>>(gpq, dgq, B * tiles, C);
        gain_combine<<<(C + 255) / 256, 256, 0, stream>>>(gpk, dgk, B * tiles, C);
    }
    return launch_status();
}

}  // namespace
}  // namespace sana

using namespace sana;

extern "C" {

int sana_linattn_backward(const void* q, const void* k, const void* v, const float* gq,
                          const float* gk, const void* dout, void* dq, void* dk, void* dv,
                          float* dgq, float* dgk, int64_t B, int64_t N, int C, int H, float eps,
                          sana_dtype dtype, void* workspace, size_t ws_bytes,
                          cudaStream_t stream) {
    return backward_impl(q, k, v, gq, gk, dout, dq, dk, dv, dgq, dgk, B, N, C, H, eps, dtype,
                         workspace, ws_bytes, stream, nullptr);
}

int sana_linattn_backward_with_state(const void* q, const void* k, const void* v,
                                     const float* gq, const float* gk, const float* kv,
                                     const void* dout, void* dq, void* dk, void* dv, float* dgq,
                                     float* dgk, int64_t B, int64_t N, int C, int H, float eps,
                                     sana_dtype dtype, void* workspace, size_t ws_bytes,
                                     cudaStream_t stream) {
    if (!kv && B > 0 && N > 0) return SANA_EINVAL;
    return backward_impl(q, k, v, gq, gk, dout, dq, dk, dv, dgq, dgk, B, N, C, H, eps, dtype,
                         workspace, ws_bytes, stream, kv);
}

int sana_linattn_forward_causal(const void* q, const void* k, const void* v, const float* gq,
                                const float* gk, void* out, int64_t B, int64_t N, int C, int H,
                                float eps, sana_dtype dtype, void* workspace, size_t ws_bytes,
                                cudaStream_t stream) {
    int rc;
    if ((rc = check_dims(B, N, C, H)) != SANA_OK) return rc;
    if ((rc = check_eps(eps)) != SANA_OK) return rc;
    if ((rc = check_gains(gq, gk)) != SANA_OK) return rc;
    if (dtype != SANA_BF16 && dtype != SANA_F32) return SANA_EINVAL;
    if (B == 0 || N == 0) return SANA_OK;
    if ((rc = validate_qkv(q, k, v, out, B, N, C, dtype)) != SANA_OK) return rc;
    const int64_t S = (N + kCausalChunk - 1) / kCausalChunk;
    const size_t need = sana_linattn_workspace_bytes(B, N, C, H, 2);
    if ((rc = validate_ws(workspace, ws_bytes, need)) != SANA_OK) return rc;
    const size_t bytes = (size_t)B * N * C * elem_size(dtype);
    if (overlaps(workspace, need, out, bytes) || overlaps(workspace, need, q, bytes) ||
        overlaps(workspace, need, k, bytes) || overlaps(workspace, need, v, bytes))
        return SANA_EINVAL;
    if (S > 0x7fffffffLL) return SANA_EUNSUPPORTED;
    float* part = (float*)workspace;
    const dim3 g1((unsigned)S, H, (unsigned)B);
    const int norm = gk != nullptr;
    if (tc_path(dtype, C) && (!norm || (aligned(gq, 16) && aligned(gk, 16))))
        return launch_causal_tc(q, k, v, gq, gk, out, B, N, C, H, eps, workspace, stream);
    if (dtype == SANA_BF16) {
        kv_partial_simt<bf16><<<g1, 128, 0, stream>>>((const bf16*)k, (const bf16*)v, gk, part, N,
                                                      H, C, C, (int)S, kCausalChunk, eps, norm);
        causal_scan<<<(unsigned)(B * H), 256, 0, stream>>>(part, (int)S);
        causal_apply_simt<bf16><<<g1, kCausalChunk, 0, stream>>>(
            (const bf16*)q, (const bf16*)k, (const bf16*)v, gq, gk, part, (bf16*)out, N, H,
            (int)S, eps, norm);
    } else {
        kv_partial_simt<float><<<g1, 128, 0, stream>>>((const float*)k, (const float*)v, gk, part,
                                                       N, H, C, C, (int)S, kCausalChunk, eps,
                                                       norm);
        causal_scan<<<(unsigned)(B * H), 256, 0, stream>>>(part, (int)S);
        causal_apply_simt<float><<<g1, kCausalChunk, 0, stream>>>(
            (const float*)q, (const float*)k, (const float*)v, gq, gk, part, (float*)out, N, H,
            (int)S, eps, norm);
    }
    return launch_status();
}

const char* sana_linattn_strerror(int status) {
    switch (status) {
        case SANA_OK: return "success";
        case SANA_EINVAL: return "invalid argument (shape, NULL pointer, eps, dtype or overlap)";
        case SANA_EALIGN: return "pointer misaligned (16 B tensors, 256 B workspace, 4 B gains)";
        case SANA_EUNSUPPORTED: return "unsupported configuration (head dim must be 32)";
        case SANA_EWORKSPACE: return "workspace missing or smaller than required";
        case SANA_ECUDA: return "CUDA launch or runtime error";
        case SANA_ESCRATCH:
            return "problem needs more scratch than the static 16 MiB array of "
                   "sana_linattn_forward_noalloc (use sana_linattn_forward with a workspace)";
        default: return "unknown status";
    }
}

int sana_linattn_kv_state(const void* k, const void* v, const float* gk, float* kv, int64_t B,
                          int64_t N, int C, int H, float eps, sana_dtype dtype, void* workspace,
                          size_t ws_bytes, cudaStream_t stream) {
    int rc;
    if ((rc = check_dims(B, N, C, H)) != SANA_OK) return rc;
    if ((rc = check_eps(eps)) != SANA_OK) return rc;
    if (dtype != SANA_BF16 && dtype != SANA_F32) return SANA_EINVAL;
    if (gk && !aligned(gk, 4)) return SANA_EALIGN;
    if (B == 0) return SANA_OK;
    if (!kv) return SANA_EINVAL;
    if (!aligned(kv, 16)) return SANA_EALIGN;
    if (N == 0) {
        return cudaMemsetAsync(kv, 0, (size_t)B * H * kStateFloats * sizeof(float), stream) ==
                       cudaSuccess ? SANA_OK : SANA_ECUDA;
    }
    if (!k || !v) return SANA_EINVAL;
    if (!aligned(k, 16) || !aligned(v, 16)) return SANA_EALIGN;
    const WsLayout L = ws_layout(B, N, C, H, false);
    if ((rc = validate_ws(workspace, ws_bytes, L.total)) != SANA_OK) return rc;
    const size_t in_bytes = (size_t)B * N * C * elem_size(dtype);
    const size_t kv_bytes = (size_t)B * H * kStateFloats * sizeof(float);
    if (overlaps(kv, kv_bytes, k, in_bytes) || overlaps(kv, kv_bytes, v, in_bytes))
        return SANA_EINVAL;
    float* part = (float*)((char*)workspace + L.part_off);
    if (tc_path(dtype, C)) {
        PersistPlan1 pl{};
        if ((rc = launch_partials_tc(k, v, gk, part, B, N, C, H, eps, stream, &pl)) != SANA_OK ||
            (rc = launch_combine_tc(part, kv, B, H, pl, stream)) != SANA_OK)
            return rc;
    } else if (dtype == SANA_BF16) {
        launch_state<bf16>((const bf16*)k, (const bf16*)v, gk, part, kv, B, N, H, C, C, eps,
                           make_plan(B, N, H), stream);
    } else {
        launch_state<float>((const float*)k, (const float*)v, gk, part, kv, B, N, H, C, C, eps,
                            make_plan(B, N, H), stream);
    }
    return launch_status();
}

int sana_linattn_apply(const void* q, const float* gq, const float* kv, void* out, int64_t B,
                       int64_t N, int C, int H, float eps, sana_dtype dtype,
                       cudaStream_t stream) {
    int rc;
    if ((rc = check_dims(B, N, C, H)) != SANA_OK) return rc;
    if ((rc = check_eps(eps)) != SANA_OK) return rc;
    if (dtype != SANA_BF16 && dtype != SANA_F32) return SANA_EINVAL;
    if (gq && !aligned(gq, 4)) return SANA_EALIGN;
    if (B == 0 || N == 0) return SANA_OK;
    if (!q || !kv || !out) return SANA_EINVAL;
    if (!aligned(q, 16) || !aligned(out, 16) || !aligned(kv, 16)) return SANA_EALIGN;
    const size_t bytes = (size_t)B * N * C * elem_size(dtype);
    if (overlaps(out, bytes, q, bytes) ||
        overlaps(out, bytes, kv, (size_t)B * H * kStateFloats * sizeof(float)))
        return SANA_EINVAL;
    if (tc_path(dtype, C)) {
        if ((rc = launch_apply_tc(q, gq, kv, nullptr, nullptr, out, B, N, C, H, eps, stream)) !=
            SANA_OK)
            return rc;
    } else if (dtype == SANA_BF16) {
        launch_apply<bf16, bf16>((const bf16*)q, gq, kv, (bf16*)out, B, N, H, C, C, eps, stream);
    } else {
        launch_apply<float, float>((const float*)q, gq, kv, (float*)out, B, N, H, C, C, eps,
                                   stream);
    }
    return launch_status();
}

int sana_linattn_forward(const void* q, const void* k, const void* v, const float* gq,
                         const float* gk, void* out, int64_t B, int64_t N, int C, int H,
                         float eps, sana_dtype dtype, void* workspace, size_t ws_bytes,
                         cudaStream_t stream) {
    int rc;
    if ((rc = check_dims(B, N, C, H)) != SANA_OK) return rc;
    if ((rc = check_eps(eps)) != SANA_OK) return rc;
    if ((rc = check_gains(gq, gk)) != SANA_OK) return rc;
    if (dtype != SANA_BF16 && dtype != SANA_F32) return SANA_EINVAL;
    if (B == 0 || N == 0) return SANA_OK;
    if ((rc = validate_qkv(q, k, v, out, B, N, C, dtype)) != SANA_OK) return rc;
    const WsLayout L = ws_layout(B, N, C, H, false);
    if ((rc = validate_ws(workspace, ws_bytes, L.total)) != SANA_OK) return rc;
    const size_t bytes = (size_t)B * N * C * elem_size(dtype);
    if (overlaps(workspace, L.total, out, bytes) || overlaps(workspace, L.total, q, bytes) ||
        overlaps(workspace, L.total, k, bytes) || overlaps(workspace, L.total, v, bytes))
        return SANA_EINVAL;
    const Plan p = make_plan(B, N, H);
    float* part = (float*)((char*)workspace + L.part_off);
    float* kv = (float*)((char*)workspace + L.kv_off);
    if (tc_path(dtype, C) && short_path(B, N, H)) {
        if ((rc = launch_short_tc(q, k, v, gq, gk, out, B, N, C, H, eps, stream)) != SANA_OK)
            return rc;
    } else if (tc_path(dtype, C)) {
        PersistPlan1 pl{};
        if ((rc = launch_partials_tc(k, v, gk, part, B, N, C, H, eps, stream, &pl)) != SANA_OK ||
            (rc = launch_apply_tc(q, gq, nullptr, part, &pl, out, B, N, C, H, eps, stream)) !=
                SANA_OK)
            return rc;
    } else if (dtype == SANA_BF16) {
        launch_state<bf16>((const bf16*)k, (const bf16*)v, gk, part, kv, B, N, H, C, C, eps, p,
                           stream);
        launch_apply<bf16, bf16>((const bf16*)q, gq, kv, (bf16*)out, B, N, H, C, C, eps, stream);
    } else {
        launch_state<float>((const float*)k, (const float*)v, gk, part, kv, B, N, H, C, C, eps, p,
                            stream);
        launch_apply<float, float>((const float*)q, gq, kv, (float*)out, B, N, H, C, C, eps,
                                   stream);
    }
    return launch_status();
}

int sana_linattn_forward_kernels(int64_t B, int64_t N, int C, int H, sana_dtype dtype) {
    int rc;
    if ((rc = check_dims(B, N, C, H)) != SANA_OK) return rc;
    if (dtype != SANA_BF16 && dtype != SANA_F32) return SANA_EINVAL;
    if (B == 0 || N == 0) return 0;
    if (!tc_path(dtype, C)) return 3;
    return short_path(B, N, H) ? 1 : 2;
}

int sana_linattn_forward_pass1(const void* k, const void* v, const float* gk, int64_t B,
                               int64_t N, int C, int H, float eps, void* workspace,
                               size_t ws_bytes, cudaStream_t stream) {
    int rc;
    if ((rc = check_dims(B, N, C, H)) != SANA_OK) return rc;
    if ((rc = check_eps(eps)) != SANA_OK) return rc;
    if (gk && !aligned(gk, 4)) return SANA_EALIGN;
    if (!tc_path(SANA_BF16, C)) return SANA_EUNSUPPORTED;
    if (B == 0 || N == 0) return SANA_OK;
    if (!k || !v) return SANA_EINVAL;
    if (!aligned(k, 16) || !aligned(v, 16)) return SANA_EALIGN;
    const WsLayout L = ws_layout(B, N, C, H, false);
    if ((rc = validate_ws(workspace, ws_bytes, L.total)) != SANA_OK) return rc;
    const size_t bytes = (size_t)B * N * C * 2;
    if (overlaps(workspace, L.total, k, bytes) || overlaps(workspace, L.total, v, bytes))
        return SANA_EINVAL;
    float* part = (float*)((char*)workspace + L.part_off);
    if ((rc = launch_partials_tc(k, v, gk, part, B, N, C, H, eps, stream, nullptr)) != SANA_OK)
        return rc;
    return launch_status();
}

int sana_linattn_forward_pass2(const void* q, const float* gq, void* out, int64_t B, int64_t N,
                               int C, int H, float eps, void* workspace, size_t ws_bytes,
                               cudaStream_t stream) {
    int rc;
    if ((rc = check_dims(B, N, C, H)) != SANA_OK) return rc;
    if ((rc = check_eps(eps)) != SANA_OK) return rc;
    if (gq && !aligned(gq, 4)) return SANA_EALIGN;
    if (!tc_path(SANA_BF16, C)) return SANA_EUNSUPPORTED;
    if (B == 0 || N == 0) return SANA_OK;
    if (!q || !out) return SANA_EINVAL;
    if (!aligned(q, 16) || !aligned(out, 16)) return SANA_EALIGN;
    const WsLayout L = ws_layout(B, N, C, H, false);
    if ((rc = validate_ws(workspace, ws_bytes, L.total)) != SANA_OK) return rc;
    const size_t bytes = (size_t)B * N * C * 2;
    if (overlaps(out, bytes, q, bytes) || overlaps(workspace, L.total, q, bytes) ||
        overlaps(workspace, L.total, out, bytes))
        return SANA_EINVAL;
    const int P = persistent_ctas();
    if (P == 0) return SANA_ECUDA;
    const PersistPlan1 pl = make_plan_p1(B, N, H, P);     // the plan pass 1 used
    float* part = (float*)((char*)workspace + L.part_off);
    if ((rc = launch_apply_tc(q, gq, nullptr, part, &pl, out, B, N, C, H, eps, stream)) != SANA_OK)
        return rc;
    return launch_status();
}

int sana_linattn_qkv_fused(const void* x, const void* Wqkv, const float* gq, const float* gk,
                           void* out, int64_t B, int64_t N, int C, int H, float eps,
                           void* workspace, size_t ws_bytes, cudaStream_t stream) {
    int rc;
    if ((rc = check_dims(B, N, C, H)) != SANA_OK) return rc;
    if ((rc = check_eps(eps)) != SANA_OK) return rc;
    if ((rc = check_gains(gq, gk)) != SANA_OK) return rc;
    if (B == 0 || N == 0) return SANA_OK;
    if (!x || !Wqkv || !out) return SANA_EINVAL;
    if (!aligned(x, 16) || !aligned(Wqkv, 16) || !aligned(out, 16)) return SANA_EALIGN;
    const size_t xb = (size_t)B * N * C * 2, wb = (size_t)C * 3 * C * 2;
    if (overlaps(out, xb, x, xb) || overlaps(out, xb, Wqkv, wb)) return SANA_EINVAL;
    const WsLayout L = ws_layout(B, N, C, H, true);
    if ((rc = validate_ws(workspace, ws_bytes, L.total)) != SANA_OK) return rc;
    if (overlaps(workspace, L.total, out, xb) || overlaps(workspace, L.total, x, xb) ||
        overlaps(workspace, L.total, Wqkv, wb))
        return SANA_EINVAL;
    if (B * (int64_t)((H + 3) / 4) > 65535 * 65535LL) return SANA_EUNSUPPORTED;
    float* part = (float*)((char*)workspace + L.part_off);
    float* kv = (float*)((char*)workspace + L.kv_off);
    int* counters = (int*)((char*)workspace + L.counters_off);
    if ((rc = launch_fused<false>(x, Wqkv, nullptr, nullptr, gq, gk, out, counters, part, kv, B, N,
                                  C, H, eps, stream)) != SANA_OK)
        return rc;
    return launch_status();
}

int sana_linattn_qkv_fused_w8a8(const int8_t* xq, const float* sx, const int8_t* Wq,
                                const float* sw, const float* gq, const float* gk, void* out,
                                int64_t B, int64_t N, int C, int H, float eps, void* workspace,
                                size_t ws_bytes, cudaStream_t stream) {
    int rc;
    if ((rc = check_dims(B, N, C, H)) != SANA_OK) return rc;
    if ((rc = check_eps(eps)) != SANA_OK) return rc;
    if ((rc = check_gains(gq, gk)) != SANA_OK) return rc;
    if (B == 0 || N == 0) return SANA_OK;
    if (!xq || !sx || !Wq || !sw || !out) return SANA_EINVAL;
    if (!aligned(xq, 16) || !aligned(Wq, 16) || !aligned(out, 16) || !aligned(sx, 4) ||
        !aligned(sw, 4))
        return SANA_EALIGN;
    const size_t xb = (size_t)B * N * C, wb = (size_t)C * 3 * C, ob = (size_t)B * N * C * 2;
    if (overlaps(out, ob, xq, xb) || overlaps(out, ob, Wq, wb) ||
        overlaps(out, ob, sx, (size_t)B * N * 4) || overlaps(out, ob, sw, (size_t)3 * C * 4))
        return SANA_EINVAL;
    const WsLayout L = ws_layout(B, N, C, H, true);
    if ((rc = validate_ws(workspace, ws_bytes, L.total)) != SANA_OK) return rc;
    if (overlaps(workspace, L.total, out, ob) || overlaps(workspace, L.total, xq, xb) ||
        overlaps(workspace, L.total, Wq, wb))
        return SANA_EINVAL;
    if (B * (int64_t)((H + 3) / 4) > 65535 * 65535LL) return SANA_EUNSUPPORTED;
    float* part = (float*)((char*)workspace + L.part_off);
    float* kv = (float*)((char*)workspace + L.kv_off);
    int* counters = (int*)((char*)workspace + L.counters_off);
    if ((rc = launch_fused<true>(xq, Wq, sx, sw, gq, gk, out, counters, part, kv, B, N, C, H, eps,
                                 stream)) != SANA_OK)
        return rc;
    return launch_status();
}

int sana_quantize_rows_i8(const void* x, sana_dtype dtype, int8_t* xq, float* scales,
                          int64_t rows, int cols, cudaStream_t stream) {
    if (rows < 0 || cols <= 0 || cols % 8 != 0) return SANA_EINVAL;
    if (dtype != SANA_BF16 && dtype != SANA_F32) return SANA_EINVAL;
    if (rows == 0) return SANA_OK;
    if (!x || !xq || !scales) return SANA_EINVAL;
    if (!aligned(x, dtype == SANA_BF16 ? 16 : 32) || !aligned(xq, 8) || !aligned(scales, 4))
        return SANA_EALIGN;
    const size_t in = (size_t)rows * cols * elem_size(dtype), qb = (size_t)rows * cols;
    if (overlaps(xq, qb, x, in) || overlaps(scales, (size_t)rows * 4, x, in) ||
        overlaps(scales, (size_t)rows * 4, xq, qb))
        return SANA_EINVAL;
    if ((rows + 7) / 8 > 0x7fffffffLL) return SANA_EUNSUPPORTED;
    const dim3 grid((unsigned)((rows + 7) / 8));
    if (dtype == SANA_BF16)
        quantize_rows_i8<bf16><<<grid, 256, 0, stream>>>((const bf16*)x, xq, scales, rows, cols);
    else
        quantize_rows_i8<float><<<grid, 256, 0, stream>>>((const float*)x, xq, scales, rows, cols);
    return launch_status();
}

int sana_quantize_cols_i8(const void* w, sana_dtype dtype, int8_t* wq, float* scales, int64_t K,
                          int cols, cudaStream_t stream) {
    if (K < 0 || cols <= 0) return SANA_EINVAL;
    if (dtype != SANA_BF16 && dtype != SANA_F32) return SANA_EINVAL;
    if (K == 0) return SANA_OK;
    if (!w || !wq || !scales) return SANA_EINVAL;
    if (!aligned(w, elem_size(dtype)) || !aligned(scales, 4)) return SANA_EALIGN;
    const size_t in = (size_t)K * cols * elem_size(dtype), qb = (size_t)K * cols;
    if (overlaps(wq, qb, w, in) || overlaps(scales, (size_t)cols * 4, w, in) ||
        overlaps(scales, (size_t)cols * 4, wq, qb))
        return SANA_EINVAL;
    const dim3 grid((unsigned)((cols + 31) / 32)), block(32, 8);
    if (dtype == SANA_BF16)
        quantize_cols_i8<bf16><<<grid, block, 0, stream>>>((const bf16*)w, wq, scales, K, cols);
    else
        quantize_cols_i8<float><<<grid, block, 0, stream>>>((const float*)w, wq, scales, K, cols);
    return launch_status();
}

int sana_linattn_forward_noalloc(const void* q, const void* k, const void* v, const float* gq,
                                 const float* gk, void* out, int64_t B, int64_t N, int C, int H,
                                 float eps, sana_dtype dtype, cudaStream_t stream) {
    int rc;
    if ((rc = check_dims(B, N, C, H)) != SANA_OK) return rc;
    if (B > 0 && N > 0 && ws_layout(B, N, C, H, false).total > kNoAllocScratchBytes)
        return SANA_ESCRATCH;
    void* scratch = nullptr;
    if ((rc = noalloc_scratch(&scratch)) != SANA_OK) return rc;
    // Same kernels and plan as sana_linattn_forward; the scratch takes the place
    // of the caller's workspace.  Every scratch byte the forward path reads it
    // has written earlier in the same call, so nothing needs clearing.
    return sana_linattn_forward(q, k, v, gq, gk, out, B, N, C, H, eps, dtype, scratch,
                                kNoAllocScratchBytes, stream);
}

int sana_linattn_selftest_launch_failure(cudaStream_t stream) {
    // 2048 threads in one block is above the per-block limit: the runtime rejects
    // the launch (nothing reaches the GPU) and the error surfaces like any other
    // launch failure of the library.
    launch_failure_selftest<<<1, 2048, 0, stream>>>();
    return launch_status();
}

int sana_linattn_selftest_wait_timeout(int64_t limit_us, cudaStream_t stream) {
    if (limit_us < 0 || limit_us > 10000000) return SANA_EINVAL;
    wait_timeout_selftest<<<1, 32, 0, stream>>>((uint64_t)limit_us * 1000ull, 999);
    return launch_status();
}

int sana_linattn_device_error(int* code, int* site, int clear) {
    int c = 0, where = 0;
    if (cudaMemcpyFromSymbol(&c, g_device_error, sizeof(int)) != cudaSuccess ||
        cudaMemcpyFromSymbol(&where, g_device_error_site, sizeof(int)) != cudaSuccess)
        return SANA_ECUDA;
    if (code) *code = c;
    if (site) *site = where;
    if (clear) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)) != cudaSuccess ||
            cudaMemcpyToSymbol(g_device_error_site, &zero, sizeof(int)) != cudaSuccess)
            return SANA_ECUDA;
    }
    return SANA_OK;
}

}  // extern "C"

// ============================================================================ Mix-FFN
namespace sana {
namespace {

// A row-major (rows, cols) bf16 matrix seen by TMA as 2-D (cols, rows), boxes of
// 64 columns (128 bytes) x box_rows rows, 128-byte swizzle; out-of-range reads
// are zeros (ragged M, N and K tails).
bool make_tmap_rowmajor(CUtensorMap* m, const void* base, int64_t rows, int64_t cols,
                        uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    const cuuint32_t box[2] = {64u, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

// u (B, Hs, Ws, 2F) bf16 as 4-D (2F, Ws, Hs, B), boxes of 32 channels x 34 tokens x
// 1 row x 1 batch, no swizzle; coordinates outside the grid read as zeros.
bool make_tmap_grid(CUtensorMap* m, const void* u, int64_t B, int Hs, int Ws, int F) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t ch = 2 * (cuuint64_t)F;
    const cuuint64_t dims[4] = {ch, (cuuint64_t)Ws, (cuuint64_t)Hs, (cuuint64_t)B};
    const cuuint64_t strides[3] = {ch * 2, ch * 2 * Ws, ch * 2 * Ws * Hs};
    const cuuint32_t box[4] = {(cuuint32_t)dw::kCh, (cuuint32_t)dw::kBoxTok, 1, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(u), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

// CTAs of the persistent GEMM: one per SM (its shared memory and 512 TMEM columns
// allow no second).  0 on failure.
int gemm_ctas() {
    static int ctas[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    if (ctas[dev]) return ctas[dev];
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        sms <= 0)
        return 0;
    if (cudaFuncSetAttribute(gemm_bias_bf16_2sm, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             g2::kSmemBytes) != cudaSuccess)
        return 0;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, gemm_bias_bf16_2sm, g2::kThreads,
                                                      g2::kSmemBytes) != cudaSuccess ||
        per_sm < 1)
        return 0;
    ctas[dev] = sms;
    return sms;
}

int check_gemm(const void* A, const void* W, const float* bias, const void* D, int64_t M, int K,
               int Nc) {
    if (M < 0 || K <= 0 || Nc <= 0 || K % 8 != 0 || Nc % 8 != 0) return SANA_EINVAL;
    if (M >= ((int64_t)1 << 31)) return SANA_EUNSUPPORTED;
    if (M == 0) return SANA_OK;
    if (!A || !W || !D) return SANA_EINVAL;
    if (!aligned(A, 16) || !aligned(W, 16) || !aligned(D, 16)) return SANA_EALIGN;
    if (bias && !aligned(bias, 4)) return SANA_EALIGN;
    const size_t nd = (size_t)M * Nc * 2;
    if (overlaps(D, nd, A, (size_t)M * K * 2) || overlaps(D, nd, W, (size_t)K * Nc * 2) ||
        overlaps(D, nd, bias, (size_t)Nc * 4))
        return SANA_EINVAL;
    return SANA_OK;
}

int launch_gemm(const void* A, const void* W, const float* bias, void* D, int64_t M, int K, int Nc,
                cudaStream_t st) {
    if (M == 0) return SANA_OK;
    const int P = gemm_ctas();
    if (!P) return SANA_EUNSUPPORTED;
    CUtensorMap ta, tw;
    if (!make_tmap_rowmajor(&ta, A, M, K, g2::kBM) || !make_tmap_rowmajor(&tw, W, K, Nc, g2::kBK))
        return SANA_ECUDA;
    GemmArgs a{};
    a.bias = bias;
    a.d = (bf16*)D;
    a.M = M;
    a.Nc = Nc;
    a.K = K;
    a.mb = (int)((M + g2::kBM - 1) / g2::kBM);
    a.nb = (Nc + g2::kBN - 1) / g2::kBN;
    // pairs of SMs (clusters of two CTAs), one 256 x 256 tile at a time
    const int64_t tiles2 = (int64_t)((M + 2 * g2::kBM - 1) / (2 * g2::kBM)) * a.nb;
    const int64_t pairs = tiles2 < P / 2 ? tiles2 : P / 2;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(2 * pairs));
    cfg.blockDim = dim3(g2::kThreads);
    cfg.dynamicSmemBytes = g2::kSmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, gemm_bias_bf16_2sm, ta, tw, a) != cudaSuccess) return SANA_ECUDA;
    return launch_status();
}

int check_grid(int64_t B, int Hs, int Ws, int F) {
    if (B < 0 || Hs < 0 || Ws < 0 || F <= 0 || F % 8 != 0) return SANA_EINVAL;
    if (B > 65535 || Hs >= (1 << 24) || Ws >= (1 << 24)) return SANA_EUNSUPPORTED;
    if ((F + dw::kCh - 1) / dw::kCh > (1 << 30)) return SANA_EUNSUPPORTED;
    return SANA_OK;
}

int launch_dwconv(const void* u, const float* wdw, const float* bdw, void* h, int64_t B, int Hs,
                  int Ws, int F, int gate, cudaStream_t st) {
    if (B == 0 || Hs == 0 || Ws == 0) return SANA_OK;
    CUtensorMap tu;
    if (!make_tmap_grid(&tu, u, B, Hs, Ws, F)) return SANA_ECUDA;
    const dim3 grid((unsigned)((F + dw::kCh - 1) / dw::kCh), (unsigned)((Ws + dw::kTX - 1) / dw::kTX),
                    (unsigned)B);
    if (gate == SANA_GATE_SIGMOID)
        dwconv3x3_glu<kGateSigmoid><<<grid, dw::kThreads, 0, st>>>(tu, wdw, bdw, (bf16*)h, Hs, Ws, F);
    else
        dwconv3x3_glu<kGateSilu><<<grid, dw::kThreads, 0, st>>>(tu, wdw, bdw, (bf16*)h, Hs, Ws, F);
    return launch_status();
}

int check_dwconv(const void* u, const float* wdw, const float* bdw, const void* h, int64_t B,
                 int Hs, int Ws, int F, int gate) {
    int rc;
    if ((rc = check_grid(B, Hs, Ws, F)) != SANA_OK) return rc;
    if (gate != SANA_GATE_SIGMOID && gate != SANA_GATE_SILU) return SANA_EINVAL;
    if (B == 0 || Hs == 0 || Ws == 0) return SANA_OK;
    if (!u || !wdw || !h) return SANA_EINVAL;
    if (!aligned(u, 16) || !aligned(h, 16)) return SANA_EALIGN;
    if (!aligned(wdw, 4) || (bdw && !aligned(bdw, 4))) return SANA_EALIGN;
    const size_t tok = (size_t)B * Hs * Ws;
    if (overlaps(h, tok * F * 2, u, tok * 2 * F * 2) ||
        overlaps(h, tok * F * 2, wdw, (size_t)2 * F * 9 * 4) ||
        overlaps(h, tok * F * 2, bdw, (size_t)2 * F * 4))
        return SANA_EINVAL;
    return SANA_OK;
}

struct MixLayout {
    size_t u_off, h_off, total;
};

MixLayout mix_layout(int64_t B, int Hs, int Ws, int F) {
    const size_t tok = (size_t)B * Hs * Ws;
    MixLayout l{};
    l.u_off = 0;
    l.h_off = align_up(tok * 2 * F * 2, 256);
    l.total = align_up(l.h_off + tok * F * 2, 256);
    return l;
}

}  // namespace
}  // namespace sana

extern "C" {

int sana_gemm_bias_bf16(const void* A, const void* W, const float* bias, void* D, int64_t M, int K,
                        int Nc, cudaStream_t stream) {
    int rc;
    if ((rc = check_gemm(A, W, bias, D, M, K, Nc)) != SANA_OK) return rc;
    return launch_gemm(A, W, bias, D, M, K, Nc, stream);
}

int sana_mixffn_dwconv_glu(const void* u, const float* wdw, const float* bdw, void* h, int64_t B,
                           int Hs, int Ws, int F, int gate, cudaStream_t stream) {
    int rc;
    if ((rc = check_dwconv(u, wdw, bdw, h, B, Hs, Ws, F, gate)) != SANA_OK) return rc;
    return launch_dwconv(u, wdw, bdw, h, B, Hs, Ws, F, gate, stream);
}

size_t sana_mixffn_workspace_bytes(int64_t B, int Hs, int Ws, int C, int F) {
    if (check_grid(B, Hs, Ws, F) != SANA_OK || C <= 0 || C % 8 != 0) return 0;
    if (B == 0 || Hs == 0 || Ws == 0) return 0;
    return mix_layout(B, Hs, Ws, F).total;
}

int sana_mixffn_forward(const void* x, const void* W1, const float* b1, const float* wdw,
                        const float* bdw, const void* W2, const float* b2, void* y, int64_t B,
                        int Hs, int Ws, int C, int F, int gate, void* workspace, size_t ws_bytes,
                        cudaStream_t stream) {
    int rc;
    if ((rc = check_grid(B, Hs, Ws, F)) != SANA_OK) return rc;
    if (C <= 0 || C % 8 != 0) return SANA_EINVAL;
    if (gate != SANA_GATE_SIGMOID && gate != SANA_GATE_SILU) return SANA_EINVAL;
    if (B == 0 || Hs == 0 || Ws == 0) return SANA_OK;
    const int64_t M = B * (int64_t)Hs * Ws;
    if (M >= ((int64_t)1 << 31)) return SANA_EUNSUPPORTED;
    if (!x || !W1 || !wdw || !W2 || !y) return SANA_EINVAL;
    const MixLayout l = mix_layout(B, Hs, Ws, F);
    if ((rc = validate_ws(workspace, ws_bytes, l.total)) != SANA_OK) return rc;
    uint8_t* ws = (uint8_t*)workspace;
    void* U = ws + l.u_off;
    void* Hg = ws + l.h_off;
    const void* args[] = {x, W1, b1, wdw, bdw, W2, b2, y};
    const size_t sizes[] = {(size_t)M * C * 2, (size_t)C * 2 * F * 2, (size_t)2 * F * 4,
                            (size_t)2 * F * 9 * 4, (size_t)2 * F * 4, (size_t)F * C * 2,
                            (size_t)C * 4, (size_t)M * C * 2};
    for (int i = 0; i < 8; ++i)
        if (overlaps(workspace, l.total, args[i], sizes[i])) return SANA_EINVAL;
    if ((rc = check_gemm(x, W1, b1, U, M, C, 2 * F)) != SANA_OK) return rc;
    if ((rc = check_dwconv(U, wdw, bdw, Hg, B, Hs, Ws, F, gate)) != SANA_OK) return rc;
    if ((rc = check_gemm(Hg, W2, b2, y, M, F, C)) != SANA_OK) return rc;
    for (int i = 0; i < 6; ++i)
        if (overlaps(y, sizes[7], args[i], sizes[i])) return SANA_EINVAL;
    if ((rc = launch_gemm(x, W1, b1, U, M, C, 2 * F, stream)) != SANA_OK) return rc;
    if ((rc = launch_dwconv(U, wdw, bdw, Hg, B, Hs, Ws, F, gate, stream)) != SANA_OK) return rc;
    return launch_gemm(Hg, W2, b2, y, M, F, C, stream);
}

}  // extern "C"

// C ABI of libgconv.so (declared in include/gconv.h): argument validation,
// geometry, per-shape kernel planning, the GroupNorm workspace, and the two
// entry points of the FP32 NCHW conv2d forward and the fused
// conv -> bias -> scale -> sigmoid -> GroupNorm chain.
#include <algorithm>
#include <cmath>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "gconv.h"
#include "gconv_internal.h"

using namespace gconv;

namespace {

constexpr int kMaxThreads = 256;
constexpr size_t kSmemBudget = 100 * 1024;   // keep two CTAs per SM where possible
constexpr size_t kSmemMax = 227 * 1024;
constexpr int kBarFloats = 32;               // shared memory reserved for mbarriers

enum ForceMode : int {
    kForceAuto = 0, kForceDirect = 1, kForceGeneric = 2, kForceCpAsync = 3, kForceIgemm = 4,
    kForceBlocked = 5, kForceStream = 6, kForceIgemmSplit = 7, kForceIgemmFused = 8, kForceWinograd = 9
};
std::atomic<int> g_force{kForceAuto};
std::atomic<int> g_force_kt{0};   // channels per thread forced for the direct kernels (0: planner's rule)


// Convolution geometry.  stride, pad and dil are the H-axis values; sw, pw
// and dw the W-axis ones (equal to them for the symmetric entry points).
struct Shape {
    int N, C, H, W, K, R, S, stride, pad, dil, groups;
    int cpg, kpg, P, Q;
    int sw, pw, dw;
    bool square() const { return stride == sw && pad == pw && dil == dw; }
};

long long out_extent(long long in, long long k, long long s, long long p, long long d) {
    long long span = in + 2 * p - d * (k - 1) - 1;
    if (span < 0) return 0;
    return span / s + 1;
}

gconv_status_t make_shape_ex(Shape &s, int N, int C, int H, int W, int K, int R, int S, int sh, int sw, int ph,
                             int pw, int dh, int dw, int groups) {
    if (N < 1 || C < 1 || H < 1 || W < 1 || K < 1 || R < 1 || S < 1) return GCONV_ERR_INVALID_ARG;
    if (sh < 1 || sw < 1 || ph < 0 || pw < 0 || dh < 1 || dw < 1 || groups < 1) return GCONV_ERR_INVALID_ARG;
    if (C % groups != 0 || K % groups != 0) return GCONV_ERR_INVALID_ARG;
    long long P = out_extent(H, R, sh, ph, dh);
    long long Q = out_extent(W, S, sw, pw, dw);
    if (P < 1 || Q < 1 || P > 0x7fffffff || Q > 0x7fffffff) return GCONV_ERR_INVALID_ARG;
    // index arithmetic: per-plane offsets fit in int64 comfortably; keep the
    // element counts below 2^62 and the staged-tile arithmetic in int
    if ((long long)N * C * H * W >= (1LL << 62) || (long long)N * K * P * Q >= (1LL << 62))
        return GCONV_ERR_INVALID_ARG;
    if ((long long)H * W >= (1LL << 31) || P * Q >= (1LL << 31)) return GCONV_ERR_UNSUPPORTED;
    s = {N, C, H, W, K, R, S, sh, ph, dh, groups, C / groups, K / groups, (int)P, (int)Q, sw, pw, dw};
    return GCONV_OK;
}

gconv_status_t make_shape(Shape &s, int N, int C, int H, int W, int K, int R, int S, int stride, int pad,
                          int dil, int groups) {
    return make_shape_ex(s, N, C, H, W, K, R, S, stride, stride, pad, pad, dil, dil, groups);
}

// Per-shape kernel choices measured on B200 (dispatch_table.json, compiled in
// at build time): the fastest of the streaming direct kernel, the blocked
// direct kernel and the implicit GEMM, with the direct kernels' channels per
// thread, timed per shape; shapes not in the table follow the planner's rules.
enum TableFamily : int { kTabStream = 1, kTabBlocked = 2, kTabIgemm = 3, kTabWinograd = 4, kTabIgemmFused = 5 };
struct DispatchEntry {
    int key[12];   // N, C, H, W, K, R, S, stride, pad, dilation, groups, chain
    int family;
    int kt;
};
const DispatchEntry kDispatchTable[] = {
#include "gconv_dispatch_table.inc"
    {{0}, 0, 0}   // end marker
};

// The measured choice for a shape with equal axes, or nullptr.
const DispatchEntry *table_choice(const Shape &s, bool chain) {
    if (!s.square()) return nullptr;
    const int key[12] = {s.N, s.C, s.H, s.W, s.K, s.R, s.S, s.stride, s.pad, s.dil, s.groups, chain ? 1 : 0};
    for (const DispatchEntry *e = kDispatchTable; e->family; ++e)
        if (!std::memcmp(e->key, key, sizeof(key))) return e;
    return nullptr;
}

int match_geom(const Shape &s) {
    if (s.dil != 1 || !s.square()) return kDirectGeneric;
    if (s.R == 3 && s.S == 3 && s.stride == 1 && s.pad == 1) return kGeom3x3s1p1;
    if (s.R == 3 && s.S == 3 && s.stride == 1 && s.pad == 0) return kGeom3x3s1p0;
    if (s.R == 3 && s.S == 3 && s.stride == 2 && s.pad == 1) return kGeom3x3s2p1;
    if (s.R == 5 && s.S == 9 && s.stride == 1 && s.pad == 0) return kGeom5x9s1p0;
    if (s.R == 1 && s.S == 1 && s.stride == 1 && s.pad == 0) return kGeom1x1s1p0;
    return kDirectGeneric;
}

const char *geom_name(int geom) {
    switch (geom) {
        case kGeom3x3s1p1: return "direct_3x3s1p1";
        case kGeom3x3s1p0: return "direct_3x3s1p0";
        case kGeom3x3s2p1: return "direct_3x3s2p1";
        case kGeom5x9s1p0: return "direct_5x9s1p0";
        case kGeom1x1s1p0: return "direct_1x1s1p0";
        default: return "direct_generic";
    }
}

const char *geom_name_stream(int geom) {
    switch (geom) {
        case kGeom3x3s1p1: return "direct_stream_3x3s1p1";
        case kGeom3x3s1p0: return "direct_stream_3x3s1p0";
        case kGeom3x3s2p1: return "direct_stream_3x3s2p1";
        case kGeom5x9s1p0: return "direct_stream_5x9s1p0";
        case kGeom1x1s1p0: return "direct_stream_1x1s1p0";
        default: return "direct_generic";
    }
}

const char *geom_name_tma(int geom) {
    switch (geom) {
        case kGeom3x3s1p1: return "direct_tma_3x3s1p1";
        case kGeom3x3s1p0: return "direct_tma_3x3s1p0";
        case kGeom3x3s2p1: return "direct_tma_3x3s2p1";
        case kGeom5x9s1p0: return "direct_tma_5x9s1p0";
        case kGeom1x1s1p0: return "direct_tma_1x1s1p0";
        default: return "direct_generic";
    }
}

int env_int(const char *name);   // positive integer from the environment, else 0

bool compat(int a, int b) { return a % b == 0 || b % a == 0; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int ceil_div(long long a, long long b) { return (int)((a + b - 1) / b); }

// A complete launch plan for the direct kernel (blocked or streaming).
struct DirectPlan {
    DirectParams prm;
    int geom, KT;
    dim3 grid;        // streaming: grid.x is set at launch from the occupancy
    int threads;
    size_t smem;
    int stream = 0;   // 1: direct_stream_kernel
};

int sm_count() {
    static const int n = [] {
        int dev = 0, v = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) {
            cudaGetLastError();
            return 148;
        }
        return v;
    }();
    return n;
}

// Choose the CTA tile for a direct-kernel launch.  Returns false when no tile
// fits the shared-memory limit (the shape is then unsupported by this family).
bool plan_direct(const Shape &s, bool chain, int gn_groups, int geom, bool x_vec, DirectPlan &pl, int kt_req = 0) {
    const bool fast = geom != kDirectGeneric;
    const int kgn = chain ? s.K / gn_groups : 1;
    DirectParams &p = pl.prm;
    std::memset(&p, 0, sizeof(p));

    // channels per thread: the largest of 8, 4, 2, 1 dividing kpg (and, for
    // the chain, nesting with the GroupNorm group width) that still gives the
    // GPU about 128 threads per SM (the best geometric mean over the 80-shape
    // sweep among 128, 192, 320 and 512).  A thread's KT channels share every
    // input value it loads, but on small problems parallelism wins.
    int KT = 1;
    if (fast) {
        static const int force_tgt = env_int("GCONV_DIRECT_THREADS_PER_SM");
        const long long want = (long long)sm_count() * (force_tgt > 0 ? force_tgt : kMaxThreads / 2);
        for (int c : {8, 4, 2, 1}) {
            if (s.kpg % c != 0 || (chain && !compat(kgn, c))) continue;
            KT = c;
            const long long threads =
                (long long)s.N * (s.K / c) * ceil_div(s.P, direct_rpt(c)) * ceil_div(s.Q, 4);
            if (threads >= want) break;
        }
        if (kt_req > 0 && s.kpg % kt_req == 0 && (!chain || compat(kgn, kt_req))) KT = kt_req;
    }
    const int RPT = fast ? direct_rpt(KT) : direct_rpt(1);
    if (!fast) KT = 1;

    const int qchunks = ceil_div(s.Q, 4);
    int n_qt = ceil_div(qchunks, 32);
    int CX = ceil_div(qchunks, n_qt);

    // channel slices per CTA
    const int m = s.kpg / KT;
    int KZ = 1;
    for (int z = 1; z <= m; ++z)
        if (m % z == 0 && KT * z <= 32 && CX * z <= kMaxThreads && (!chain || compat(kgn, KT * z))) KZ = z;

    const int strips = ceil_div(s.P, RPT);
    auto pick_ry = [&](int ry_cap, int &n_pt_out) {
        int ry_max = std::max(1, std::min(ry_cap, kMaxThreads / (CX * KZ)));
        n_pt_out = ceil_div(strips, ry_max);
        return ceil_div(strips, n_pt_out);
    };
    int n_pt = 1;
    int RY = pick_ry(strips, n_pt);

    // conv groups per CTA (only when a CTA already holds all channels of a group)
    auto pick_gb = [&](int gb_cap) {
        int gb = 1;
        if (s.kpg / (KT * KZ) == 1) {
            const int per = CX * RY * KZ;
            for (int gcand = 1; gcand <= std::min(s.groups, gb_cap); ++gcand) {
                if (s.groups % gcand) continue;
                if (per * gcand > kMaxThreads) break;
                if (chain && !compat(kgn, gcand * s.kpg)) continue;
                gb = gcand;
            }
        }
        return gb;
    };
    int GB = pick_gb(s.groups);

    // Small problems: split the work until the grid covers about two CTAs per
    // SM (GCONV_DIRECT_CTAS_PER_SM overrides): fewer groups per CTA, then fewer
    // rows, then fewer channel slices.
    static const int ctas_per_sm = [] {
        const int v = env_int("GCONV_DIRECT_CTAS_PER_SM");
        return v > 0 ? v : 2;
    }();
    const long long target = (long long)ctas_per_sm * sm_count();
    auto ctas = [&]() {
        return (long long)s.N * (s.kpg / (KT * KZ)) * (s.groups / GB) * n_qt * n_pt;
    };
    for (int guard = 0; guard < 64 && ctas() < target; ++guard) {
        if (GB > 1) {
            GB = pick_gb(GB - 1);
        } else if (RY > 1) {
            RY = pick_ry((RY + 1) / 2, n_pt);
        } else if (KZ > 1) {
            int z = KZ - 1;
            while (z > 1 && (m % z != 0 || (chain && !compat(kgn, KT * z)))) --z;
            KZ = z;
            RY = pick_ry(strips, n_pt);
            GB = 1;
        } else {
            break;
        }
    }
    const int TP = RY * RPT;
    const int KB = KT * KZ;
    const int n_kb = s.kpg / KB;
    const int KBtot = GB * KB;
    if (chain && !compat(kgn, KBtot)) return false;

    const int RS = s.R * s.S;
    int IHt = 0, PC = 0, pitch = 0;
    if (fast) {
        IHt = (TP - 1) * s.stride + (s.R - 1) * s.dil + 1;
        PC = (CX - 1) * s.stride + direct_fast_window_chunks(geom);
        int pcp = PC;
        while (((pcp - CX * s.stride) % 8 + 8) % 8 != 0) ++pcp;
        pitch = 4 * pcp;
    }
    auto w_floats_for = [&](int cc) -> size_t { return ((size_t)cc * RS * KBtot + 3) / 4 * 4; };
    auto x_off_for = [&](int cc) -> size_t { return kBarFloats + (w_floats_for(cc) + 31) / 32 * 32; };
    auto smem_for = [&](int cc) -> size_t {
        size_t xf = fast ? (size_t)GB * cc * IHt * pitch : 0;
        return (x_off_for(cc) + xf) * sizeof(float);
    };
    int cchunk = s.cpg;
    while (cchunk > 1 && smem_for(cchunk) > kSmemBudget) cchunk = (cchunk + 1) / 2;
    size_t smem = smem_for(cchunk);
    const int nsp = CX * RY;
    const size_t st_bytes = chain ? (kBarFloats + (size_t)3 * KBtot * nsp) * sizeof(float) : 0;

    // TMA staging: one pass over all input channels, aligned rows, boxes
    // within the 256-element limit; rows fetched in bands of ~16.
    int tma = 0, nb = 1, bh = IHt;
    size_t pstride = (size_t)IHt * pitch;
    const int planes = GB * s.cpg;
    // box rows padded to 128 bytes so every TMA destination is 128-byte aligned
    const int tpc = (PC + 7) / 8 * 8;
    if (fast && x_vec && cchunk == s.cpg && 4 * tpc <= 256 && planes <= 256) {
        static const int band_rows = [] {
            const char *e = std::getenv("GCONV_DIRECT_BAND_ROWS");
            return e ? std::max(1, std::atoi(e)) : 16;
        }();
        nb = std::min(8, std::max(1, (IHt + band_rows - 1) / band_rows));
        bh = (IHt + nb - 1) / nb;
        nb = (IHt + bh - 1) / bh;
        const size_t tpitch = 4 * (size_t)tpc;
        const size_t tps = (size_t)nb * bh * tpitch;
        const size_t tsmem = (x_off_for(cchunk) + planes * tps) * sizeof(float);
        if (bh <= 256 && tsmem <= kSmemMax) {
            tma = 1;
            PC = tpc;
            pitch = (int)tpitch;
            pstride = tps;
            smem = tsmem;
        }
    }
    if (st_bytes > smem) smem = st_bytes;
    if (smem > kSmemMax) return false;

    p.N = s.N; p.C = s.C; p.H = s.H; p.W = s.W; p.K = s.K; p.R = s.R; p.S = s.S;
    p.stride = s.stride; p.pad = s.pad; p.dil = s.dil; p.groups = s.groups;
    p.sw = s.sw; p.pw = s.pw; p.dw = s.dw;
    p.cpg = s.cpg; p.kpg = s.kpg; p.P = s.P; p.Q = s.Q;
    p.CX = CX; p.RY = RY; p.KZ = KZ; p.GB = GB;
    p.TP = TP; p.TQ = 4 * CX; p.KB = KB; p.KBtot = KBtot;
    p.n_qt = n_qt; p.n_pt = n_pt; p.n_kb = n_kb;
    p.IHt = IHt; p.PC = PC; p.pitch = pitch; p.cchunk = cchunk;
    p.w_floats = (int)w_floats_for(cchunk);
    p.x_off = (int)x_off_for(cchunk);
    p.pstride = (int)pstride;
    p.tma = tma;
    p.nb = nb;
    p.bh = bh;
    p.gn_groups = chain ? gn_groups : 0;
    p.kgn = kgn;
    p.n_sp = n_qt * n_pt;
    p.slots_k = (chain && KBtot < kgn) ? kgn / KBtot : 1;
    p.slots = p.slots_k * p.n_sp;

    const long long gy = (long long)n_kb * (s.groups / GB);
    const long long gx = (long long)n_qt * n_pt;
    if (gx > 0x7fffffffLL || gy > 65535 || s.N > 65535) return false;
    pl.grid = dim3((unsigned)gx, (unsigned)gy, (unsigned)s.N);
    pl.threads = (CX * RY * KZ * GB + 31) / 32 * 32;
    pl.smem = smem;
    pl.geom = geom;
    pl.KT = KT;
    return true;
}

// Plan for the streaming direct kernel (plain and affine epilogues, fast
// geometries, rows TMA can describe, one pass over a group's input channels).
// A work item is a blocked-kernel tile; its input (GB*cpg planes x IHt rows x
// 4*tpc columns, one TMA box) and its weight slice form one ring stage.
// Returns false when the shape does not fit this variant.
bool plan_stream(const Shape &s, int geom, bool x_vec, DirectPlan &pl, int kt_req = 0) {
    if (geom == kDirectGeneric || !x_vec) return false;
    DirectParams &p = pl.prm;
    std::memset(&p, 0, sizeof(p));
    // channels per thread: the blocked kernel's rule
    int KT = 1;
    const long long want = (long long)sm_count() * (kMaxThreads / 2);
    for (int c : {8, 4, 2, 1}) {
        if (s.kpg % c != 0) continue;
        KT = c;
        if ((long long)s.N * (s.K / c) * ceil_div(s.P, direct_rpt(c)) * ceil_div(s.Q, 4) >= want) break;
    }
    if (kt_req > 0 && s.kpg % kt_req == 0) KT = kt_req;
    const int RPT = direct_rpt(KT);
    const int nch = direct_fast_window_chunks(geom);
    const int qchunks = ceil_div(s.Q, 4);
    int n_qt = ceil_div(qchunks, 32), CX = 0, tpc = 0;
    // staged row: exactly the 16-byte chunks the item's threads read.  One TMA
    // box per item lands at the stage base, so the row pitch needs only the
    // box's 16-byte granularity.  Padding rows to 128 bytes doubled the stage
    // of 28-column planes (36 -> 64 floats) and left one CTA per SM; padding
    // only where it costs at most an eighth (aligned shared loads on 112-column
    // planes) measured no faster.  GCONV_STREAM_PAD_ROWS: 0 (default) never
    // pad, 1 always, 2 when cheap.
    static const int pad_rows = env_int("GCONV_STREAM_PAD_ROWS");
    for (;; ++n_qt) {   // column tiles until the staged row fits one 256-element box row
        CX = ceil_div(qchunks, n_qt);
        tpc = (CX - 1) * s.stride + nch;
        const int padded = (tpc + 7) / 8 * 8;
        if (pad_rows == 1 || (pad_rows == 2 && 8 * padded <= 9 * tpc)) tpc = padded;
        if (4 * tpc <= 256) break;
    }
    n_qt = ceil_div(qchunks, CX);
    const int CXP = CX <= 4 ? CX : (CX + 7) / 8 * 8;
    const int m = s.kpg / KT;
    int KZ = 1;
    for (int z = 1; z <= m; ++z)
        if (m % z == 0 && KT * z <= 32 && CXP * z <= kMaxThreads) KZ = z;
    const int strips = ceil_div(s.P, RPT);
    int n_pt = 1;
    auto pick_ry = [&](int cap) {
        const int ry_max = std::max(1, std::min(cap, kMaxThreads / (CXP * KZ)));
        n_pt = ceil_div(strips, ry_max);
        return ceil_div(strips, n_pt);
    };
    int RY = pick_ry(strips);
    auto pick_gb = [&](int cap) {
        int gb = 1;
        if (s.kpg / (KT * KZ) == 1)
            for (int gc = 1; gc <= std::min(s.groups, cap); ++gc) {
                if (s.groups % gc) continue;
                if (CXP * RY * KZ * gc > kMaxThreads || gc * s.cpg > 256) break;
                gb = gc;
            }
        return gb;
    };
    int GB = pick_gb(s.groups);
    // enough items per SM that the last round of items is a small part of the
    // work: fewer groups, rows, then slices per item.  2 per SM by default; 8
    // for large problems at one or two channels per thread, where a CTA's last
    // item otherwise weighs 1/3 of its run (measured 6-11% faster on the
    // 51 MB two-channel shapes; smaller problems and wider channel blocks lose).
    // GCONV_STREAM_ITEMS_PER_SM overrides.
    static const int per_sm_env = env_int("GCONV_STREAM_ITEMS_PER_SM");
    const double problem_mb = 4.0 * ((double)s.N * s.C * s.H * s.W + (double)s.N * s.K * s.P * s.Q) / 1e6;
    const int per_sm = per_sm_env > 0 ? per_sm_env : (KT <= 2 && problem_mb >= 40.0 ? 8 : 2);
    const long long target = (long long)per_sm * sm_count();
    auto items = [&]() { return (long long)s.N * (m / KZ) * (s.groups / GB) * n_qt * n_pt; };
    for (int guard = 0; guard < 64 && items() < target; ++guard) {
        if (GB > 1) {
            GB = pick_gb(GB - 1);
        } else if (RY > 1) {
            RY = pick_ry((RY + 1) / 2);
        } else if (KZ > 1) {
            int z = KZ - 1;
            while (z > 1 && m % z != 0) --z;
            KZ = z;
            RY = pick_ry(strips);
        } else {
            break;
        }
    }
    const int TP = RY * RPT;
    const int KB = KT * KZ;
    const int IHt = (TP - 1) * s.stride + (s.R - 1) * s.dil + 1;
    auto stage_of = [&](int gb) {
        return ((size_t)gb * s.cpg * IHt * 4 * tpc + ((size_t)s.cpg * s.R * s.S * gb * KB + 31) / 32 * 32) *
               sizeof(float);
    };
    // stages up to GCONV_STREAM_STAGE_KB (default 96): fewer packed groups per
    // item beyond it
    static const int stage_kb = [] {
        const int v = env_int("GCONV_STREAM_STAGE_KB");
        return v > 0 ? v : 96;
    }();
    while (GB > 1 && stage_of(GB) > (size_t)stage_kb * 1024) GB = pick_gb(GB - 1);
    const int KBtot = GB * KB;
    const int planes = GB * s.cpg;
    if (IHt > 256 || planes > 256 || items() > 0x7fffffffLL) return false;
    const size_t x_floats = (size_t)planes * IHt * 4 * tpc;   // 16-byte multiple: weights follow
    // stages 128-byte aligned (the TMA destination of each item)
    const size_t stage_floats = (x_floats + (size_t)s.cpg * s.R * s.S * KBtot + 31) / 32 * 32;
    const size_t stage_bytes = stage_floats * sizeof(float);
    if (stage_bytes > 96 * 1024) return false;
    // ring of 2 to 4 stages in about 64 KB per CTA (GCONV_STREAM_RING_KB
    // overrides, GCONV_STREAM_STAGES fixes the depth).  Larger budgets measured
    // no better: 108 KB for the 2 CTAs per SM that two or more channels per
    // thread allow (+0.4% on the large shapes, 6% slower on small ones), and 3
    // stages of a large item at one CTA per SM (5-18% slower).
    static const int force_stages = env_int("GCONV_STREAM_STAGES");
    static const int ring_kb = env_int("GCONV_STREAM_RING_KB");
    const size_t ring = (size_t)(ring_kb > 0 ? ring_kb : 64) * 1024;
    int S = (int)std::max<size_t>(2, std::min<size_t>(4, ring / stage_bytes));
    if (force_stages >= 2 && force_stages <= 4 && kStreamHeaderBytes + (size_t)force_stages * stage_bytes <= 227 * 1024)
        S = force_stages;

    p.N = s.N; p.C = s.C; p.H = s.H; p.W = s.W; p.K = s.K; p.R = s.R; p.S = s.S;
    p.stride = s.stride; p.pad = s.pad; p.dil = s.dil; p.groups = s.groups;
    p.sw = s.sw; p.pw = s.pw; p.dw = s.dw;
    p.cpg = s.cpg; p.kpg = s.kpg; p.P = s.P; p.Q = s.Q;
    p.CX = CX; p.CXP = CXP; p.RY = RY; p.KZ = KZ; p.GB = GB;
    p.TP = TP; p.TQ = 4 * CX; p.KB = KB; p.KBtot = KBtot;
    p.n_qt = n_qt; p.n_pt = n_pt; p.n_kb = m / KZ;
    p.IHt = IHt; p.PC = tpc; p.pitch = 4 * tpc; p.cchunk = s.cpg;
    p.pstride = IHt * 4 * tpc;
    p.tma = 1;
    p.n_items = (int)items();
    p.stages = S;
    p.stage_floats = (int)stage_floats;
    p.sw_off = (int)x_floats;
    pl.geom = geom;
    pl.KT = KT;
    pl.threads = (CXP * RY * KZ * GB + 31) / 32 * 32 + 32;
    pl.smem = kStreamHeaderBytes + (size_t)S * stage_bytes;
    pl.grid = dim3(0);
    pl.stream = 1;
    return true;
}

// Winograd F(2x2, 3x3) plan: 3x3, stride 1, dilation 1, equal padding on both
// axes, at least 2 channels per group and per thread (KT = 4, else 2).
struct WinoPlan {
    WinoParams prm;
    int KT;
    dim3 grid;
    int threads;
    size_t smem;
};

bool plan_winograd(const Shape &s, WinoPlan &pl) {
    if (s.R != 3 || s.S != 3 || s.stride != 1 || s.dil != 1 || !s.square() || s.cpg < 2) return false;
    const int KT = s.kpg % 4 == 0 ? 4 : (s.kpg % 2 == 0 ? 2 : 0);
    if (!KT) return false;
    WinoParams &p = pl.prm;
    std::memset(&p, 0, sizeof(p));
    int TX = std::min(16, (s.Q + 1) / 2), TY = std::min(8, (s.P + 1) / 2);
    const int m = s.kpg / KT;
    int KZ = 1;
    auto smem_of = [&](int tx, int ty, int kz) {
        const size_t u = (size_t)s.cpg * 16 * kz * KT;
        return (u + (size_t)s.cpg * (2 * ty + 2) * (2 * tx + 2)) * sizeof(float);
    };
    for (;;) {
        KZ = 1;
        for (int z = 1; z <= m; ++z)
            if (m % z == 0 && TX * TY * z <= 256 && smem_of(TX, TY, z) <= 100 * 1024) KZ = z;
        if (smem_of(TX, TY, KZ) <= 227 * 1024) break;
        if (TY > 1) TY = (TY + 1) / 2;
        else if (TX > 1) TX = (TX + 1) / 2;
        else return false;
    }
    p.N = s.N; p.C = s.C; p.H = s.H; p.W = s.W; p.K = s.K; p.P = s.P; p.Q = s.Q; p.pad = s.pad;
    p.cpg = s.cpg; p.kpg = s.kpg; p.groups = s.groups;
    p.TX = TX; p.TY = TY; p.KZ = KZ; p.KB = KZ * KT;
    p.n_qt = ceil_div(s.Q, 2 * TX);
    p.n_pt = ceil_div(s.P, 2 * TY);
    p.n_kb = s.kpg / p.KB;
    p.pitch = 2 * TX + 2;
    p.u_floats = s.cpg * 16 * p.KB;
    const long long gx = (long long)p.n_qt * p.n_pt, gy = (long long)s.groups * p.n_kb;
    if (gx > 0x7fffffffLL || gy > 65535 || s.N > 65535) return false;
    pl.KT = KT;
    pl.grid = dim3((unsigned)gx, (unsigned)gy, (unsigned)s.N);
    pl.threads = (TX * TY * KZ + 31) / 32 * 32;
    pl.smem = smem_of(TX, TY, KZ);
    return true;
}

// Whether the dispatcher runs a shape on the Winograd kernel: forced, or
// measured fastest (the table); never by rule.
bool use_winograd(const Shape &s, bool chain) {
    const int force = g_force.load(std::memory_order_relaxed);
    if (chain) return false;
    if (force == kForceWinograd) return true;
    if (force != kForceAuto) return false;
    const DispatchEntry *e = table_choice(s, false);
    return e && e->family == kTabWinograd;
}

// Direct-kernel plan for the current forcing mode: in automatic mode the
// measured table decides streaming vs blocked and the channels per thread;
// shapes outside it stream whenever the streaming kernel can take them.
bool choose_direct(const Shape &s, bool chain, int gn_groups, bool x_vec, DirectPlan &pl) {
    const int force = g_force.load(std::memory_order_relaxed);
    int kt = g_force_kt.load(std::memory_order_relaxed);
    bool try_stream = !chain && force != kForceBlocked && force != kForceGeneric && force != kForceCpAsync;
    if (force == kForceAuto) {
        if (const DispatchEntry *e = table_choice(s, chain)) {
            if (e->family == kTabBlocked) try_stream = false;
            kt = e->kt;
        }
    }
    const DispatchEntry *te = force == kForceAuto ? table_choice(s, chain) : nullptr;
    int geom = (force == kForceGeneric) ? (int)kDirectGeneric : match_geom(s);
    if (force == kForceCpAsync) x_vec = false;
    if (try_stream && plan_stream(s, geom, x_vec, pl, kt)) {
        // outside the table, stream only where it measured faster: problems
        // moving at least 24 MB with at most 4 channels per thread (small ones
        // are latency-bound, where the blocked kernel's per-band waits win)
        const double mb = 4.0 * ((double)s.N * s.C * s.H * s.W + (double)s.N * s.K * s.P * s.Q) / 1048576.0;
        if (force != kForceAuto || te || (pl.KT <= 4 && mb >= 24.0)) return true;
    }
    if (force == kForceStream) return false;
    pl.stream = 0;
    if (plan_direct(s, chain, gn_groups, geom, x_vec, pl, kt)) return true;
    if (geom != kDirectGeneric && force == kForceAuto)
        return plan_direct(s, chain, gn_groups, kDirectGeneric, x_vec, pl);
    return false;
}

// Per-thread caches for repeated calls of the plain convolution: the last
// few direct plans by shape (planning walks several tile candidates), and the
// last TMA descriptor by input pointer and box (encoding goes through the
// driver).  Keys hold everything the cached value depends on.
struct DirectKey {
    int v[14];
    int x_vec, force, force_kt, dev, sms;
    bool operator==(const DirectKey &o) const { return std::memcmp(this, &o, sizeof(*this)) == 0; }
};

bool cached_direct_plan(const Shape &s, bool x_vec, DirectPlan &pl) {
    struct Entry {
        DirectKey key;
        DirectPlan plan;
        bool valid;
    };
    thread_local Entry cache[4] = {};
    thread_local int next = 0;
    DirectKey k;
    std::memset(&k, 0, sizeof(k));
    const int vals[14] = {s.N, s.C, s.H, s.W, s.K, s.R, s.S, s.stride, s.pad, s.dil, s.groups, s.sw, s.pw, s.dw};
    std::memcpy(k.v, vals, sizeof(vals));
    k.x_vec = x_vec ? 1 : 0;
    k.force = g_force.load(std::memory_order_relaxed);
    k.force_kt = g_force_kt.load(std::memory_order_relaxed);
    if (cudaGetDevice(&k.dev) != cudaSuccess) return false;
    k.sms = sm_count();
    for (const Entry &e : cache)
        if (e.valid && e.key == k) {
            pl = e.plan;
            return true;
        }
    if (!choose_direct(s, false, 1, x_vec, pl)) return false;
    cache[next] = Entry{k, pl, true};
    next = (next + 1) % 4;
    return true;
}

bool cached_x_tensor_map(TensorMap *tm, const float *x, long long planes, int H, int W, int box_w, int box_h,
                         int box_planes = 1) {
    struct Entry {
        const float *x;
        long long planes;
        int H, W, box_w, box_h, box_planes, dev;
        TensorMap tm;
        bool valid;
    };
    thread_local Entry last = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    if (last.valid && last.x == x && last.planes == planes && last.H == H && last.W == W && last.box_w == box_w &&
        last.box_h == box_h && last.box_planes == box_planes && last.dev == dev) {
        *tm = last.tm;
        return true;
    }
    if (!make_x_tensor_map(tm, x, planes, H, W, box_w, box_h, box_planes)) return false;
    last = Entry{x, planes, H, W, box_w, box_h, box_planes, dev, *tm, true};
    return true;
}

// Fill the pointer-dependent fields and the TMA descriptor of a plan; a map
// the driver rejects falls back to cp.async staging.
bool finish_plan(const Shape &s, bool chain, int gn_groups, const float *x, float *y, DirectPlan &pl,
                 TensorMap &tm) {
    DirectParams &p = pl.prm;
    p.vec_in = (s.W % 4 == 0) && aligned16(x);
    p.vec2_in = !p.vec_in && (s.W % 2 == 0) && (reinterpret_cast<uintptr_t>(x) & 7u) == 0;
    p.vec_out = (s.Q % 4 == 0) && aligned16(y);
    std::memset(&tm, 0, sizeof(tm));
    if (pl.stream) {
        // one box per work item: 4*tpc columns x IHt rows x GB*cpg planes
        if (cached_x_tensor_map(&tm, x, (long long)s.N * s.C, s.H, s.W, p.pitch, p.IHt, p.GB * s.cpg)) return true;
        // a map the CUDA driver rejects: the blocked kernel with cp.async staging
        DirectPlan again;
        if (!plan_direct(s, chain, gn_groups, pl.geom, false, again)) return false;
        again.stream = 0;
        again.prm.vec_in = p.vec_in;
        again.prm.vec2_in = p.vec2_in;
        again.prm.vec_out = p.vec_out;
        pl = again;
        return true;
    }
    if (p.tma && !cached_x_tensor_map(&tm, x, (long long)s.N * s.C, s.H, s.W, 4 * p.PC, p.bh)) {
        DirectPlan again;
        if (!plan_direct(s, chain, gn_groups, pl.geom, false, again)) return false;
        again.prm.vec_in = p.vec_in;
        again.prm.vec2_in = p.vec2_in;
        again.prm.vec_out = p.vec_out;
        pl = again;
    }
    return true;
}

// ----------------------------------------------------------------- workspace
// Device addresses cached per device are only valid in the context they were
// obtained in: after cudaDeviceReset (or a primary-context reset) the device
// gets a new context and the cached address is dropped and looked up again.
void *current_context() {
    using Fn = int (*)(void **);
    static Fn fn = [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess) {
            cudaGetLastError();
            return (Fn) nullptr;
        }
        return reinterpret_cast<Fn>(ptr);
    }();
    void *ctx = nullptr;
    if (!fn || fn(&ctx) != 0) return nullptr;
    return ctx;
}

struct Workspace {
    void *ptr = nullptr;
    size_t bytes = 0;
    void *ctx = nullptr;
};
constexpr int kMaxDevices = 64;
Workspace g_ws[kMaxDevices];
std::mutex g_ws_mutex;

gconv_status_t ensure_workspace(size_t bytes, cudaStream_t stream, void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GCONV_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return GCONV_ERR_UNSUPPORTED;
    void *ctx = current_context();
    std::lock_guard<std::mutex> lock(g_ws_mutex);
    Workspace &ws = g_ws[dev];
    if (ws.ptr && ws.ctx != ctx) ws = Workspace{};   // allocated in a context that no longer exists
    if (ws.bytes >= bytes && ws.ptr) {
        *out = ws.ptr;
        return GCONV_OK;
    }
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) return GCONV_ERR_CUDA;
    if (cs != cudaStreamCaptureStatusNone) return GCONV_ERR_WORKSPACE;
    size_t want = bytes < (1u << 20) ? (1u << 20) : bytes;
    if (ws.ptr) {
        if (cudaFree(ws.ptr) != cudaSuccess) return GCONV_ERR_CUDA;   // synchronises the device
        ws.ptr = nullptr;
        ws.bytes = 0;
    }
    void *p = nullptr;
    if (cudaMalloc(&p, want) != cudaSuccess) {
        cudaGetLastError();
        return GCONV_ERR_WORKSPACE;
    }
    ws.ptr = p;
    ws.bytes = want;
    ws.ctx = ctx;
    *out = p;
    return GCONV_OK;
}

size_t chain_ws_bytes(const DirectParams &p) {
    size_t part = (size_t)p.N * p.gn_groups * p.slots * sizeof(float4);
    size_t stats = (size_t)p.N * p.gn_groups * sizeof(float2);
    return (part + 255) / 256 * 256 + stats;
}

// ----------------------------------------------------------------- implicit GEMM
struct IgemmPlan {
    IgemmParams prm;
    dim3 grid;
    size_t smem;
    size_t off_xl, off_wh, off_wl, off_part, off_stats, ws_bytes;
    int pack = 1;     // original conv groups per GEMM group (block-diagonal weights when > 1)
};

// The same convolution with gp consecutive groups packed into one: groups/gp
// groups of gp*cpg input and gp*kpg output channels (block-diagonal weights).
Shape packed_shape(const Shape &s, int gp) {
    Shape t = s;
    t.groups = s.groups / gp;
    t.cpg = s.cpg * gp;
    t.kpg = s.kpg * gp;
    return t;
}

// Packing factor that brings a narrow group to the tensor path's 32 output
// channels (0 when the shape cannot be packed so).
int igemm_pack(const Shape &s) {
    if (s.kpg >= 32 || 32 % s.kpg != 0) return 0;
    const int gp = 32 / s.kpg;
    if (s.groups % gp != 0 || (s.cpg * gp) % 8 != 0) return 0;
    return gp;
}

size_t align256(size_t v) { return (v + 255) / 256 * 256; }

int env_int(const char *name) {
    const char *e = std::getenv(name);
    return e ? std::atoi(e) : 0;
}

// Chain design on the implicit-GEMM path (GCONV_CHAIN_DESIGN=store|recompute
// overrides): recompute runs the GEMM twice and never writes the logistic
// output; store writes it and normalizes it in a streaming pass.
bool chain_recompute(const Shape &s) {
    static const int mode = [] {
        const char *e = std::getenv("GCONV_CHAIN_DESIGN");
        if (e && !std::strcmp(e, "store")) return 0;
        if (e && !std::strcmp(e, "recompute")) return 1;
        return -1;
    }();
    if (mode >= 0) return mode == 1;
    return true;
}

// Whether the implicit GEMM stages x raw and converts it in shared memory
// outside the measured table (GCONV_IGEMM_FUSED=1 turns it on): off, since on
// the chain workload the split pass plus 8-row tiles measured faster than the
// fused variant's 6-row tiles (0.88 against 1.04 ms).
bool igemm_fused_wanted() {
    static const int v = [] {
        const char *e = std::getenv("GCONV_IGEMM_FUSED");
        return e ? std::atoi(e) : 0;
    }();
    return v != 0;
}

// Stride-1 convolutions whose groups hold a multiple of 8 input channels and
// 32/64/128/256 output channels run as an implicit GEMM on the tensor cores.
// Implicit-GEMM plan.  fused: x is staged raw by TMA and converted in shared
// memory (N = 32 only, rows 16-byte multiples), so no split pass and no x
// workspace; otherwise the split pass writes the padded operand tensors.
bool plan_igemm(const Shape &s, bool chain, int gn_groups, IgemmPlan &pl, bool fused = false) {
    if (s.stride != 1 || s.sw != 1 || s.cpg % 8 != 0 || !igemm_supported_nt(s.kpg)) return false;
    if (fused && (s.kpg != 32 || s.W % 4 != 0)) return false;
    const int kgn = chain ? s.K / gn_groups : 1;
    // chain epilogue: groups nest inside a conv group, widths 1..16 or multiples of 16
    if (chain && (s.kpg > 64 || s.kpg % kgn != 0 || (kgn > 16 && kgn % 16 != 0))) return false;
    const int NT = s.kpg;
    int COLS = 128 + (s.S - 1) * s.dw;
    COLS = (COLS + 15) / 16 * 16;   // whole 16-pixel groups of the tile box
    if (COLS > 256) return false;
    // padded split operands: every tile box starts at a 16-pixel group and a
    // non-negative row, the zero border supplies the padding
    const long long Hp = (long long)s.H + s.pad;
    const long long Wp = ((long long)s.W + s.pw + 15) / 16 * 16;
    if (Hp > 0x7fffffffLL || Wp / 16 > 0x7fffffffLL) return false;
    static const int force_th = env_int("GCONV_IGEMM_TH");
    static const int force_sa = env_int("GCONV_IGEMM_SA");
    static const int force_sb = env_int("GCONV_IGEMM_SB");
    // output rows per tile: two accumulator buffers of TH*NT columns fit TMEM.
    // The chain at 32 channels takes 7 rows: with folded tap rows it measured
    // 0.745 ms per call on the 128x8x256x256 workload against 0.787 ms at 8
    // rows and 0.766 ms at 6.
    int TH = std::max(1, std::min(8, 256 / NT));
    if (chain && NT == 32) TH = 7;
    if (force_th > 0) TH = force_th;
    if (fused) TH = igemm_fused_th();   // the fused issue loop is compiled for it (fewer rows run it unrolled less)
    TH = std::min(TH, s.P);
    const size_t limit = 227 * 1024 - igemm_header_bytes(NT, chain);
    const int COLSR = COLS + 4;                     // fused raw box: room to round the start down to 4
    // tap rows folded into one MMA (dilation 1 along H).  GCONV_IGEMM_FOLD: 0 off,
    // 1 plain convolutions only, 2 (default) the chain too.  The chain's folded
    // issue runs the kernel's general loop (its fully unrolled form measured
    // slower there): 0.745 against 0.862 ms per call unfolded.
    static const int fold_env = [] {
        const char *e = std::getenv("GCONV_IGEMM_FOLD");
        return e ? std::atoi(e) : 2;
    }();
    // (the chain's fused variant stays unfolded: folded it measured 1.06 ms
    // per call against 1.01)
    const bool fold = (fold_env == 2 && !(chain && fused)) || (fold_env == 1 && !chain);
    const int rf_pref = (fold && s.dil == 1) ? igemm_fold_rf(NT, s.R) : 1;
    int AR = 0, a_bytes = 0, b_bytes = 0, sa = 0, sb = 0, raw_bytes = 0, RF = 1, RC = s.R, BS = 0;
    // stage ring for RF folded rows and TH output rows; a folded plan keeps two
    // x stages and double-buffered (or resident) weights, else it is not taken.
    // bsl: one weight slice per tap column (when a whole chunk's does not fit)
    auto fit = [&](int rf, int th, bool bsl) {
        RF = rf;
        RC = (s.R + rf - 1) / rf;
        BS = bsl ? 1 : 0;
        // one w operand slice: (S or 1) tap columns x RF rows x 8 channels x NT
        b_bytes = 32 * (bsl ? 1 : s.S) * rf * NT;
        AR = th + (s.R - 1) * s.dil;                // staged rows serving every tap row
        if (AR > 256) return false;
        a_bytes = 32 * COLS * AR;                   // one x operand tile: 2 quads x AR x COLS x 16 B
        raw_bytes = fused ? 8 * AR * COLSR * 4 : 0;
        const size_t lim = limit - (size_t)raw_bytes;
        const int slices = s.cpg / 8 * RC * (bsl ? s.S : 1);
        sa = force_sa > 0 ? std::min(force_sa, 4) : 2;
        sb = force_sb > 0 ? std::min(force_sb, 4) : 4;
        // weights resident when every slice fits (they are then loaded once per CTA)
        if (fused && slices <= 4) sb = std::max(sb, slices);
        auto bytes = [&] { return (size_t)sa * 2 * a_bytes + (size_t)sb * 2 * b_bytes; };
        if (rf > 1) sb = std::min(sb, slices);      // no more slots than slices
        while (sb > 2 && bytes() > lim) --sb;
        while (sa > 1 && bytes() > lim) --sa;
        while (sb > 1 && bytes() > lim) --sb;
        if (bytes() > lim || (fused && sa != 2)) return false;
        return rf == 1 || (sa >= 2 && (sb >= 2 || slices <= sb));
    };
    // one slice per tap column (GCONV_IGEMM_FOLD_SLICES=1) measured 26% slower on
    // the dense 5x9 workload than one MMA per tap row: the 4-slot weight ring
    // and its per-tile reloads stall the issue; off by default
    static const bool fold_slices = env_int("GCONV_IGEMM_FOLD_SLICES") == 1;
    bool planned = rf_pref > 1 && (fit(rf_pref, TH, false) || (fold_slices && fit(rf_pref, TH, true)));
    while (!planned && TH >= 1) {
        planned = fit(1, TH, false);
        if (!planned) --TH;
    }
    if (!planned) return false;
    if (fused && (COLSR > 256 || raw_bytes <= 0)) return false;
    int tmem_cols = 32;
    while (tmem_cols < 2 * TH * NT) tmem_cols *= 2;
    if (tmem_cols > 512) return false;

    IgemmParams &p = pl.prm;
    std::memset(&p, 0, sizeof(p));
    p.N = s.N; p.C = s.C; p.H = s.H; p.W = s.W; p.K = s.K; p.R = s.R; p.S = s.S;
    p.pad = s.pad; p.dil = s.dil; p.groups = s.groups; p.cpg = s.cpg; p.kpg = s.kpg; p.P = s.P; p.Q = s.Q;
    p.pad_w = s.pw; p.dil_w = s.dw;
    p.CC8 = s.cpg / 8;
    p.RF = RF;
    p.RC = RC;
    p.bs = BS;
    p.TH = TH;
    p.COLS = COLS;
    p.Hp = (int)Hp;
    p.Wp = (int)Wp;
    p.n_qt = (s.Q + 127) / 128;
    p.n_pt = (s.P + TH - 1) / TH;
    const long long n_tiles = (long long)s.N * s.groups * p.n_qt * p.n_pt;
    if (n_tiles > 0x7fffffffLL) return false;
    p.n_tiles = (int)n_tiles;
    p.AR = AR;
    p.sa = sa;
    p.sb = sb;
    p.b_resident = p.CC8 * RC * (BS ? s.S : 1) <= sb ? 1 : 0;
    p.a_bytes = a_bytes;
    p.b_bytes = b_bytes;
    p.tmem_cols = tmem_cols;
    p.gn_groups = chain ? gn_groups : 0;
    p.kgn = kgn;
    p.slots = p.n_qt * p.n_pt * (chain ? igemm_partials_per_tile(NT, kgn) : 1);
    p.fused = fused ? 1 : 0;
    p.COLSR = fused ? COLSR : 0;
    p.raw_bytes = raw_bytes;
    p.rr = fused ? 1 : 0;
    pl.grid = dim3((unsigned)std::min<long long>(n_tiles, sm_count()));
    pl.smem = igemm_header_bytes(NT, chain) + (size_t)sa * 2 * a_bytes + (size_t)sb * 2 * b_bytes + raw_bytes;

    const size_t xbytes = fused ? 0 : (size_t)s.N * s.C * (size_t)Hp * (size_t)Wp * sizeof(float);
    const size_t wbytes = (size_t)s.K * s.cpg * RC * RF * s.S * sizeof(float);
    pl.off_xl = align256(xbytes);
    pl.off_wh = pl.off_xl + align256(xbytes);
    pl.off_wl = pl.off_wh + align256(wbytes);
    pl.off_part = pl.off_wl + align256(wbytes);
    const size_t part = chain ? (size_t)s.N * gn_groups * p.slots * sizeof(float4) : 0;
    pl.off_stats = pl.off_part + align256(part);
    pl.ws_bytes = pl.off_stats + (chain ? (size_t)s.N * gn_groups * sizeof(float2) : 0);
    return true;
}

const char *igemm_name(const IgemmPlan &ig) {
    if (ig.pack > 1) return ig.prm.fused ? "igemm_tf32_bf16x_fused_packed" : "igemm_tf32_bf16x_packed";
    return ig.prm.fused ? "igemm_tf32_bf16x_fused" : "igemm_tf32_bf16x";
}

bool force_is_igemm() {
    const int f = g_force.load(std::memory_order_relaxed);
    return f == kForceIgemm || f == kForceIgemmSplit || f == kForceIgemmFused;
}

// A fused plan stages x by TMA, which needs x 16-byte aligned: otherwise
// re-plan the split variant (returns false when that does not fit either).
bool igemm_plan_for_pointer(const Shape &s, bool chain, int gn_groups, const float *x, IgemmPlan &pl) {
    if (!pl.prm.fused || aligned16(x)) return true;
    if (g_force.load(std::memory_order_relaxed) == kForceIgemmFused) return false;
    const int gp = pl.pack;
    if (!plan_igemm(gp > 1 ? packed_shape(s, gp) : s, chain, gn_groups, pl, false)) return false;
    pl.pack = gp;
    return true;
}

// Whether the dispatcher sends a shape to the implicit GEMM.
bool use_igemm(const Shape &s, bool chain, int gn_groups, IgemmPlan &pl) {
    const int force = g_force.load(std::memory_order_relaxed);
    if (force == kForceDirect || force == kForceGeneric || force == kForceCpAsync || force == kForceBlocked ||
        force == kForceStream || force == kForceWinograd)
        return false;
    // groups narrower than the tensor path's 32 output channels run packed
    const int gp = igemm_pack(s);
    const Shape sp = gp ? packed_shape(s, gp) : s;
    pl.pack = gp ? gp : 1;
    if (force == kForceIgemmFused) return plan_igemm(sp, chain, gn_groups, pl, true);
    if (force == kForceIgemmSplit) return plan_igemm(sp, chain, gn_groups, pl, false);
    const DispatchEntry *e = force == kForceAuto ? table_choice(s, chain) : nullptr;
    const bool fused = e ? e->family == kTabIgemmFused : igemm_fused_wanted();
    if (!(fused && plan_igemm(sp, chain, gn_groups, pl, true)) && !plan_igemm(sp, chain, gn_groups, pl))
        return false;
    if (force == kForceIgemm) return true;
    if (e) return e->family == kTabIgemm || e->family == kTabIgemmFused;
    // outside the table: enough reduction depth and output channels for the tensor cores to win;
    // packed groups only where measured (the table)
    return !gp && s.cpg * s.R * s.S >= 64;
}

// Launch the split passes and the GEMM; chain additionally runs the GroupNorm
// finalize and normalize passes.
// Tensor maps over the split x operands in the workspace (x_hi, cross terms);
// for the fused variant a map over x itself ([N*C][H][W], box COLSR x AR x 8).
bool igemm_maps(const Shape &s, const IgemmPlan &pl, void *ws, TensorMap *tm, const float *x = nullptr) {
    char *base = reinterpret_cast<char *>(ws);
    const IgemmParams &p = pl.prm;
    if (p.fused) {
        std::memset(&tm[1], 0, sizeof(tm[1]));
        return x && aligned16(x) &&
               cached_x_tensor_map(&tm[0], x, (long long)s.N * s.C, s.H, s.W, p.COLSR, p.AR, 8);
    }
    const long long quads = (long long)s.N * (s.C / 4);
    return make_nc4hw4_tile_map(&tm[0], reinterpret_cast<float *>(base), quads, p.Hp, p.Wp, p.COLS, p.AR) &&
           make_nc4hw4_tile_map(&tm[1], reinterpret_cast<float *>(base + pl.off_xl), quads, p.Hp, p.Wp, p.COLS,
                                p.AR);
}

gconv_status_t run_igemm(const Shape &s, IgemmPlan &pl, const float *x, const float *w, const float *bias,
                         const float *scale, int gn_groups, const float *gamma, const float *beta, float eps,
                         float *y, void *ws, cudaStream_t stream, const TensorMap *maps = nullptr,
                         bool split_w = true) {
    char *base = reinterpret_cast<char *>(ws);
    float *xh = reinterpret_cast<float *>(base);
    float *xl = reinterpret_cast<float *>(base + pl.off_xl);
    float *wh = reinterpret_cast<float *>(base + pl.off_wh);
    float *wl = reinterpret_cast<float *>(base + pl.off_wl);
    IgemmParams &p = pl.prm;
    TensorMap own[2];
    const TensorMap *tm = maps;
    if (!tm) {
        if (!igemm_maps(s, pl, ws, own, x)) return GCONV_ERR_UNSUPPORTED;
        tm = own;
    }
    p.wh = reinterpret_cast<const float4 *>(wh);
    p.wl = reinterpret_cast<const float4 *>(wl);
    p.bias = bias;
    p.scale = scale;
    p.y = y;
    const bool chain = gn_groups > 0;
    p.gn_part = chain ? reinterpret_cast<float4 *>(base + pl.off_part) : nullptr;
    if (!p.fused && launch_split_x(x, xh, xl, s.N, s.C, s.H, s.W, s.pad, s.pw, p.Hp, p.Wp, stream) != cudaSuccess)
        return GCONV_ERR_CUDA;
    if (split_w && launch_split_w(w, wh, wl, s.K, p.cpg, s.R, s.S, p.RF, p.groups, stream, pl.pack) != cudaSuccess)
        return GCONV_ERR_CUDA;
    // the chain either stores the logistic output and normalizes it in a
    // streaming pass (store), or runs the GEMM twice: statistics only, then the
    // normalized result straight from the accumulators (recompute; y is written
    // once and the logistic output never reaches memory)
    const bool recompute = chain && chain_recompute(s);
    p.chain_mode = recompute ? 1 : 0;
    if (launch_igemm(p, tm, chain ? 1 : 0, pl.grid, pl.smem, stream) != cudaSuccess) return GCONV_ERR_CUDA;
    if (!chain) return GCONV_OK;
    GnParams g;
    g.y = y;
    g.gn_part = p.gn_part;
    g.stats = reinterpret_cast<float2 *>(base + pl.off_stats);
    g.gamma = gamma; g.beta = beta;
    g.N = s.N; g.K = s.K; g.gn_groups = gn_groups; g.kgn = s.K / gn_groups; g.slots = p.slots;
    g.PQ = (long long)s.P * s.Q;
    g.eps = eps;
    g.vec = (g.PQ % 4 == 0) && aligned16(y);
    const long long per_cta = g.vec ? 4LL * 256 * 8 : 256LL * 8;
    g.chunks = (int)std::max<long long>(1, (g.PQ + per_cta - 1) / per_cta);
    if (launch_gn_finalize(g, stream) != cudaSuccess) return GCONV_ERR_CUDA;
    if (recompute) {
        p.chain_mode = 2;
        p.gn_stats = g.stats;
        p.gamma = gamma;
        p.beta = beta;
        return launch_igemm(p, tm, 1, pl.grid, pl.smem, stream) == cudaSuccess ? GCONV_OK : GCONV_ERR_CUDA;
    }
    if (launch_gn_normalize(g, stream) != cudaSuccess) return GCONV_ERR_CUDA;
    return GCONV_OK;
}

// Images per chunk of the fused chain on the implicit-GEMM path.  With a
// budget set (GCONV_CHAIN_L2_MB), each chunk's conv output and split operands
// take about that much of the L2 cache, so the normalize pass could read the
// conv output back from L2.  Measured on B200 this loses to one pass over the
// whole batch at every budget tried (24-112 MB: 1.0-1.6 ms against 0.91 ms;
// per-chunk GEMM ramp and tail, statistics merge and launch costs outweigh
// the saved HBM traffic), so by default the whole batch is one chunk.
int chain_chunk_images(const Shape &s, const IgemmPlan &pl) {
    static const int budget_mb = env_int("GCONV_CHAIN_L2_MB");
    if (budget_mb <= 0) return s.N;
    const double per_img = 4.0 * s.K * s.P * s.Q + 8.0 * s.C * pl.prm.Hp * (double)pl.prm.Wp;
    const long long B = (long long)(budget_mb * 1048576.0 / per_img);
    return (int)std::max<long long>(1, std::min<long long>(B, s.N));
}

// The fused chain on the implicit-GEMM path, one chunk of images at a time
// (split x -> GEMM with the fused epilogue -> statistics merge -> normalize);
// the workspace holds one chunk.
gconv_status_t run_chain_igemm(const Shape &s, const IgemmPlan &full, const float *x, const float *w,
                               const float *bias, const float *scale, int gn_groups, const float *gamma,
                               const float *beta, float eps, float *y, cudaStream_t stream) {
    const int B = chain_chunk_images(s, full);
    Shape sc = s;
    sc.N = B;
    const bool fused = full.prm.fused != 0;
    const int gp = full.pack;
    IgemmPlan first;
    if (B == s.N) first = full;
    else if (!plan_igemm(gp > 1 ? packed_shape(sc, gp) : sc, true, gn_groups, first, fused)) return GCONV_ERR_UNSUPPORTED;
    first.pack = gp;
    void *ws = nullptr;
    gconv_status_t st = ensure_workspace(first.ws_bytes, stream, &ws);
    if (st != GCONV_OK) return st;
    TensorMap maps[2];   // split variant: maps over the workspace, the same for every chunk
    if (!fused && !igemm_maps(sc, first, ws, maps)) return GCONV_ERR_UNSUPPORTED;
    const long long x_img = (long long)s.C * s.H * s.W, y_img = (long long)s.K * s.P * s.Q;
    for (int n0 = 0; n0 < s.N; n0 += B) {
        const int nb = std::min(B, s.N - n0);
        if (nb == B) {
            IgemmPlan cur = first;
            st = run_igemm(sc, cur, x + n0 * x_img, w, bias, scale, gn_groups, gamma, beta, eps, y + n0 * y_img, ws,
                           stream, fused ? nullptr : maps, n0 == 0);
        } else {
            // a shorter last chunk: its own plan (workspace offsets and maps follow N)
            Shape sl = s;
            sl.N = nb;
            IgemmPlan cur;
            if (!plan_igemm(gp > 1 ? packed_shape(sl, gp) : sl, true, gn_groups, cur, fused))
                return GCONV_ERR_UNSUPPORTED;
            cur.pack = gp;
            st = run_igemm(sl, cur, x + n0 * x_img, w, bias, scale, gn_groups, gamma, beta, eps, y + n0 * y_img, ws,
                           stream);
        }
        if (st != GCONV_OK) return st;
    }
    return GCONV_OK;
}

gconv_status_t validate_ptrs(const float *x, const float *w, const float *y) {
    if (!x || !w || !y) return GCONV_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(w) | reinterpret_cast<uintptr_t>(y)) & 3u)
        return GCONV_ERR_INVALID_ARG;
    return GCONV_OK;
}

// Plain convolution, optionally with the affine + clamp epilogue.
gconv_status_t conv_fwd_shape(const Shape &s, const float *x, const float *w, const float *bias,
                              const float *aff_scale, int clamp, float lo, float hi, float *y, cudaStream_t stream) {
    gconv_status_t st;
    if ((st = validate_ptrs(x, w, y)) != GCONV_OK) return st;
    if (bias && (reinterpret_cast<uintptr_t>(bias) & 3u)) return GCONV_ERR_INVALID_ARG;
    if (aff_scale && (reinterpret_cast<uintptr_t>(aff_scale) & 3u)) return GCONV_ERR_INVALID_ARG;
    IgemmPlan ig;
    if (use_igemm(s, false, 1, ig) && igemm_plan_for_pointer(s, false, 1, x, ig)) {
        void *ws = nullptr;
        if ((st = ensure_workspace(ig.ws_bytes, stream, &ws)) != GCONV_OK) return st;
        ig.prm.aff_scale = aff_scale;
        ig.prm.clamp = clamp;
        ig.prm.lo = lo;
        ig.prm.hi = hi;
        return run_igemm(s, ig, x, w, bias, nullptr, 0, nullptr, nullptr, 0.f, y, ws, stream);
    }
    if (force_is_igemm()) return GCONV_ERR_UNSUPPORTED;
    if (use_winograd(s, false)) {
        WinoPlan wp;
        if (!plan_winograd(s, wp)) {
            if (g_force.load(std::memory_order_relaxed) == kForceWinograd) return GCONV_ERR_UNSUPPORTED;
        } else {
            WinoParams &q = wp.prm;
            q.x = x; q.w = w; q.bias = bias; q.y = y;
            q.aff_scale = aff_scale; q.clamp = clamp; q.lo = lo; q.hi = hi;
            q.vec_out = (s.Q % 2 == 0) && (reinterpret_cast<uintptr_t>(y) & 7u) == 0;
            return launch_winograd(q, wp.KT, wp.grid, wp.threads, wp.smem, stream) == cudaSuccess ? GCONV_OK
                                                                                               : GCONV_ERR_CUDA;
        }
    }
    DirectPlan pl;
    const bool x_vec = (s.W % 4 == 0) && aligned16(x);
    if (!cached_direct_plan(s, x_vec, pl)) return GCONV_ERR_UNSUPPORTED;
    TensorMap tm;
    if (!finish_plan(s, false, 1, x, y, pl, tm)) return GCONV_ERR_UNSUPPORTED;
    DirectParams &p = pl.prm;
    p.x = x; p.w = w; p.bias = bias; p.y = y;
    p.aff_scale = aff_scale;
    p.clamp = clamp;
    p.lo = lo;
    p.hi = hi;
    const cudaError_t e = pl.stream
                              ? launch_direct_stream(p, tm, pl.geom, pl.KT, sm_count(), pl.threads, pl.smem, stream)
                              : launch_direct(p, tm, pl.geom, pl.KT, 0, pl.grid, pl.threads, pl.smem, stream);
    return e == cudaSuccess ? GCONV_OK : GCONV_ERR_CUDA;
}

gconv_status_t conv_fwd(const float *x, const float *w, const float *bias, const float *aff_scale, int clamp,
                        float lo, float hi, int N, int C, int H, int W, int K, int R, int S, int stride, int pad,
                        int dilation, int groups, float *y, cudaStream_t stream) {
    Shape s;
    gconv_status_t st = make_shape(s, N, C, H, W, K, R, S, stride, pad, dilation, groups);
    if (st != GCONV_OK) return st;
    return conv_fwd_shape(s, x, w, bias, aff_scale, clamp, lo, hi, y, stream);
}

}  // namespace

extern "C" {

const char *gconv_status_string(gconv_status_t status) {
    switch (status) {
        case GCONV_OK: return "GCONV_OK";
        case GCONV_ERR_INVALID_ARG: return "GCONV_ERR_INVALID_ARG: invalid size, pointer or parameter";
        case GCONV_ERR_UNSUPPORTED: return "GCONV_ERR_UNSUPPORTED: valid shape that no kernel implements";
        case GCONV_ERR_CUDA: return "GCONV_ERR_CUDA: the CUDA runtime reported an error";
        case GCONV_ERR_WORKSPACE: return "GCONV_ERR_WORKSPACE: workspace too small and cannot grow now";
        case GCONV_ERR_TIMEOUT: return "GCONV_ERR_TIMEOUT: a bounded device wait gave up";
    }
    return "unknown gconv status";
}

const char *gconv_version(void) { return "gconv-b200 0.2.0 (sm_100a)"; }

gconv_status_t gconv_device_error_status(void) {
    int v = read_and_clear_device_error();
    int u = read_and_clear_igemm_error();
    if (v < 0 || u < 0) return GCONV_ERR_CUDA;
    return (v || u) ? GCONV_ERR_TIMEOUT : GCONV_OK;
}

gconv_status_t gconv_get_last_device_error(cudaStream_t stream) {
    if (cudaStreamSynchronize(stream) != cudaSuccess) return GCONV_ERR_CUDA;
    return gconv_device_error_status();
}

gconv_status_t gconv_selftest_wait_timeout(unsigned int spins, cudaStream_t stream) {
    if (spins < 1 || spins > (1u << 24)) return GCONV_ERR_INVALID_ARG;
    return launch_wait_timeout_probe(spins, stream) == cudaSuccess ? GCONV_OK : GCONV_ERR_CUDA;
}

gconv_status_t gconv2d_output_size(int H, int W, int R, int S, int stride, int pad, int dilation, int *P,
                                   int *Q) {
    if (!P || !Q) return GCONV_ERR_INVALID_ARG;
    Shape s;
    gconv_status_t st = make_shape(s, 1, 1, H, W, 1, R, S, stride, pad, dilation, 1);
    if (st == GCONV_ERR_UNSUPPORTED) st = GCONV_OK;   // extents are still defined
    if (st != GCONV_OK) return st;
    *P = (int)out_extent(H, R, stride, pad, dilation);
    *Q = (int)out_extent(W, S, stride, pad, dilation);
    return GCONV_OK;
}

gconv_status_t gconv_force_kernel(const char *name) {
    if (!name) return GCONV_ERR_INVALID_ARG;
    // optional ":ktN" suffix: channels per thread of the direct kernels
    char fam[32];
    int kt = 0;
    const char *colon = std::strchr(name, ':');
    const size_t n = colon ? (size_t)(colon - name) : std::strlen(name);
    if (n >= sizeof(fam)) return GCONV_ERR_INVALID_ARG;
    std::memcpy(fam, name, n);
    fam[n] = 0;
    if (colon) {
        if (std::strcmp(colon + 1, "kt1") == 0) kt = 1;
        else if (std::strcmp(colon + 1, "kt2") == 0) kt = 2;
        else if (std::strcmp(colon + 1, "kt4") == 0) kt = 4;
        else if (std::strcmp(colon + 1, "kt8") == 0) kt = 8;
        else return GCONV_ERR_INVALID_ARG;
    }
    int mode;
    if (!std::strcmp(fam, "auto")) mode = kForceAuto;
    else if (!std::strcmp(fam, "direct")) mode = kForceDirect;
    else if (!std::strcmp(fam, "generic")) mode = kForceGeneric;
    else if (!std::strcmp(fam, "direct_cpasync")) mode = kForceCpAsync;
    else if (!std::strcmp(fam, "igemm")) mode = kForceIgemm;
    else if (!std::strcmp(fam, "direct_blocked")) mode = kForceBlocked;
    else if (!std::strcmp(fam, "direct_stream")) mode = kForceStream;
    else if (!std::strcmp(fam, "igemm_split")) mode = kForceIgemmSplit;
    else if (!std::strcmp(fam, "igemm_fused")) mode = kForceIgemmFused;
    else if (!std::strcmp(fam, "winograd")) mode = kForceWinograd;
    else return GCONV_ERR_INVALID_ARG;
    if (kt && (mode == kForceAuto || mode == kForceIgemm || mode == kForceIgemmSplit || mode == kForceIgemmFused ||
               mode == kForceWinograd))
        return GCONV_ERR_INVALID_ARG;
    g_force = mode;
    g_force_kt = kt;
    return GCONV_OK;
}

const char *gconv2d_plan_name(int N, int C, int H, int W, int K, int R, int S, int stride, int pad,
                              int dilation, int groups, int chain) {
    Shape s;
    gconv_status_t st = make_shape(s, N, C, H, W, K, R, S, stride, pad, dilation, groups);
    if (st == GCONV_ERR_INVALID_ARG) return "invalid";
    if (st != GCONV_OK) return "unsupported";
    IgemmPlan ig;
    if (use_igemm(s, chain != 0, chain ? s.K : 1, ig)) return igemm_name(ig);
    WinoPlan wp;
    if (use_winograd(s, chain != 0) && plan_winograd(s, wp)) return "winograd_f2x2_3x3";
    if (g_force.load(std::memory_order_relaxed) == kForceWinograd) return "unsupported";
    DirectPlan pl;
    int gn = 1;
    if (!choose_direct(s, chain != 0, gn, s.W % 4 == 0, pl)) return "unsupported";
    if (pl.stream) return geom_name_stream(pl.geom);
    return pl.prm.tma ? geom_name_tma(pl.geom) : geom_name(pl.geom);
}

gconv_status_t gconv2d_fwd(const float *x, const float *w, const float *bias, int N, int C, int H, int W, int K,
                           int R, int S, int stride, int pad, int dilation, int groups, float *y,
                           cudaStream_t stream) {
    return conv_fwd(x, w, bias, nullptr, 0, 0.f, 0.f, N, C, H, W, K, R, S, stride, pad, dilation, groups, y, stream);
}

gconv_status_t gconv2d_fwd_ex(const float *x, const float *w, const float *bias, int N, int C, int H, int W, int K,
                              int R, int S, int stride_h, int stride_w, int pad_h, int pad_w, int dil_h, int dil_w,
                              int groups, float *y, cudaStream_t stream) {
    Shape s;
    gconv_status_t st =
        make_shape_ex(s, N, C, H, W, K, R, S, stride_h, stride_w, pad_h, pad_w, dil_h, dil_w, groups);
    if (st != GCONV_OK) return st;
    return conv_fwd_shape(s, x, w, bias, nullptr, 0, 0.f, 0.f, y, stream);
}

const char *gconv2d_plan_name_ex(int N, int C, int H, int W, int K, int R, int S, int stride_h, int stride_w,
                                 int pad_h, int pad_w, int dil_h, int dil_w, int groups) {
    Shape s;
    gconv_status_t st =
        make_shape_ex(s, N, C, H, W, K, R, S, stride_h, stride_w, pad_h, pad_w, dil_h, dil_w, groups);
    if (st == GCONV_ERR_INVALID_ARG) return "invalid";
    if (st != GCONV_OK) return "unsupported";
    IgemmPlan ig;
    if (use_igemm(s, false, 1, ig)) return igemm_name(ig);
    WinoPlan wp;
    if (use_winograd(s, false) && plan_winograd(s, wp)) return "winograd_f2x2_3x3";
    if (g_force.load(std::memory_order_relaxed) == kForceWinograd) return "unsupported";
    DirectPlan pl;
    if (!choose_direct(s, false, 1, s.W % 4 == 0, pl)) return "unsupported";
    if (pl.stream) return geom_name_stream(pl.geom);
    return pl.prm.tma ? geom_name_tma(pl.geom) : geom_name(pl.geom);
}

gconv_status_t gconv2d_affine_clamp_fwd(const float *x, const float *w, int N, int C, int H, int W, int K, int R,
                                        int S, int stride, int pad, int dilation, int groups, const float *scale,
                                        const float *shift, float lo, float hi, float *y, cudaStream_t stream) {
    if (!(lo <= hi)) return GCONV_ERR_INVALID_ARG;   // also rejects NaN bounds
    const int clamp = (lo > -INFINITY || hi < INFINITY) ? 1 : 0;
    return conv_fwd(x, w, shift, scale, clamp, lo, hi, N, C, H, W, K, R, S, stride, pad, dilation, groups, y,
                    stream);
}

size_t gconv2d_chain_workspace_size(int N, int C, int H, int W, int K, int R, int S, int stride, int pad,
                                    int dilation, int groups, int gn_groups) {
    Shape s;
    if (make_shape(s, N, C, H, W, K, R, S, stride, pad, dilation, groups) != GCONV_OK) return 0;
    if (gn_groups < 1 || K % gn_groups) return 0;
    IgemmPlan ig;
    if (use_igemm(s, true, gn_groups, ig)) {
        const int B = chain_chunk_images(s, ig);
        if (B == s.N) return ig.ws_bytes;
        Shape sc = s;
        sc.N = B;
        IgemmPlan first;
        return plan_igemm(ig.pack > 1 ? packed_shape(sc, ig.pack) : sc, true, gn_groups, first, ig.prm.fused != 0)
                   ? first.ws_bytes : 0;
    }
    DirectPlan pl;
    if (!choose_direct(s, true, gn_groups, s.W % 4 == 0, pl)) return 0;
    return chain_ws_bytes(pl.prm);
}

gconv_status_t gconv_reserve_workspace(size_t bytes) {
    void *p = nullptr;
    return ensure_workspace(bytes, nullptr, &p);
}

gconv_status_t gconv2d_bias_scale_sigmoid_groupnorm_fwd(const float *x, const float *w, const float *bias, int N,
                                                        int C, int H, int W, int K, int R, int S, int stride,
                                                        int pad, int dilation, int groups, const float *scale,
                                                        int gn_groups, const float *gamma, const float *beta,
                                                        float eps, float *y, cudaStream_t stream) {
    Shape s;
    gconv_status_t st = make_shape(s, N, C, H, W, K, R, S, stride, pad, dilation, groups);
    if (st != GCONV_OK) return st;
    if ((st = validate_ptrs(x, w, y)) != GCONV_OK) return st;
    if (!scale || !gamma || !beta) return GCONV_ERR_INVALID_ARG;
    if (gn_groups < 1 || K % gn_groups != 0) return GCONV_ERR_INVALID_ARG;
    if (!(eps >= 0.f) || eps != eps) return GCONV_ERR_INVALID_ARG;
    for (const void *q : {(const void *)bias, (const void *)scale, (const void *)gamma, (const void *)beta})
        if (q && (reinterpret_cast<uintptr_t>(q) & 3u)) return GCONV_ERR_INVALID_ARG;
    IgemmPlan ig;
    if (use_igemm(s, true, gn_groups, ig) && igemm_plan_for_pointer(s, true, gn_groups, x, ig))
        return run_chain_igemm(s, ig, x, w, bias, scale, gn_groups, gamma, beta, eps, y, stream);
    if (force_is_igemm() || g_force.load(std::memory_order_relaxed) == kForceWinograd) return GCONV_ERR_UNSUPPORTED;
    DirectPlan pl;
    const bool x_vec = (s.W % 4 == 0) && aligned16(x);
    if (!choose_direct(s, true, gn_groups, x_vec, pl)) return GCONV_ERR_UNSUPPORTED;
    TensorMap tm;
    if (!finish_plan(s, true, gn_groups, x, y, pl, tm)) return GCONV_ERR_UNSUPPORTED;
    DirectParams &p = pl.prm;
    void *ws = nullptr;
    const size_t part_bytes = ((size_t)p.N * p.gn_groups * p.slots * sizeof(float4) + 255) / 256 * 256;
    if ((st = ensure_workspace(chain_ws_bytes(p), stream, &ws)) != GCONV_OK) return st;
    p.x = x; p.w = w; p.bias = bias; p.y = y; p.scale = scale;
    p.gn_part = reinterpret_cast<float4 *>(ws);
    if (launch_direct(p, tm, pl.geom, pl.KT, 1, pl.grid, pl.threads, pl.smem, stream) != cudaSuccess)
        return GCONV_ERR_CUDA;

    GnParams g;
    g.y = y;
    g.gn_part = p.gn_part;
    g.stats = reinterpret_cast<float2 *>(reinterpret_cast<char *>(ws) + part_bytes);
    g.gamma = gamma; g.beta = beta;
    g.N = s.N; g.K = s.K; g.gn_groups = gn_groups; g.kgn = s.K / gn_groups; g.slots = p.slots;
    g.PQ = (long long)s.P * s.Q;
    g.eps = eps;
    g.vec = (g.PQ % 4 == 0) && aligned16(y);
    const long long per_cta = g.vec ? 4LL * 256 * 8 : 256LL * 8;
    g.chunks = (int)((g.PQ + per_cta - 1) / per_cta);
    if (g.chunks < 1) g.chunks = 1;
    if (launch_gn_finalize(g, stream) != cudaSuccess) return GCONV_ERR_CUDA;
    if (launch_gn_normalize(g, stream) != cudaSuccess) return GCONV_ERR_CUDA;
    return GCONV_OK;
}

}  // extern "C"

// ------------------------------------------------------------------------
// Allocation-free variant of the fused chain (gconv2d_bias_scale_sigmoid_
// groupnorm_fwd_noalloc).  Its GroupNorm partials live in a fixed array in
// device memory that every GPU loading this library reserves until process
// exit, instead of the workspace the regular entry point grows with
// cudaMalloc.  Host code must not hand the array's name to a kernel: on the
// host that name is only a stand-in, so the device address is looked up with
// cudaGetSymbolAddress once per device (with that device current) and passed
// as a pointer.
static constexpr size_t kNoAllocScratchBytes = 4u << 20;   // 4 MiB per GPU
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

void *g_noalloc_ptr[kMaxDevices];
void *g_noalloc_ctx[kMaxDevices];
std::mutex g_noalloc_mutex;

// Device address of the scratch array on the current device; the first call
// per device (and the first after the device's context was reset) performs
// the lookup.
gconv_status_t noalloc_scratch(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GCONV_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return GCONV_ERR_UNSUPPORTED;
    void *ctx = current_context();
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_ptr[dev] || g_noalloc_ctx[dev] != ctx) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) {
            cudaGetLastError();
            return GCONV_ERR_CUDA;
        }
        g_noalloc_ptr[dev] = ptr;
        g_noalloc_ctx[dev] = ctx;
    }
    *out = g_noalloc_ptr[dev];
    return GCONV_OK;
}

}  // namespace

extern "C" {

size_t gconv_noalloc_scratch_capacity(void) { return kNoAllocScratchBytes; }

gconv_status_t gconv2d_bias_scale_sigmoid_groupnorm_fwd_noalloc(
    const float *x, const float *w, const float *bias, int N, int C, int H, int W, int K, int R, int S,
    int stride, int pad, int dilation, int groups, const float *scale, int gn_groups, const float *gamma,
    const float *beta, float eps, float *y, cudaStream_t stream) {
    Shape s;
    gconv_status_t st = make_shape(s, N, C, H, W, K, R, S, stride, pad, dilation, groups);
    if (st != GCONV_OK) return st;
    if ((st = validate_ptrs(x, w, y)) != GCONV_OK) return st;
    if (!scale || !gamma || !beta) return GCONV_ERR_INVALID_ARG;
    if (gn_groups < 1 || K % gn_groups != 0) return GCONV_ERR_INVALID_ARG;
    if (!(eps >= 0.f) || eps != eps) return GCONV_ERR_INVALID_ARG;
    for (const void *q : {(const void *)bias, (const void *)scale, (const void *)gamma, (const void *)beta})
        if (q && (reinterpret_cast<uintptr_t>(q) & 3u)) return GCONV_ERR_INVALID_ARG;
    DirectPlan pl;
    const bool x_vec = (s.W % 4 == 0) && aligned16(x);
    if (!choose_direct(s, true, gn_groups, x_vec, pl)) return GCONV_ERR_UNSUPPORTED;
    TensorMap tm;
    if (!finish_plan(s, true, gn_groups, x, y, pl, tm)) return GCONV_ERR_UNSUPPORTED;
    DirectParams &p = pl.prm;
    // every partial slot and every statistics entry is written by this call
    // before it is read, so stale contents from an earlier call never leak
    if (chain_ws_bytes(p) > kNoAllocScratchBytes) return GCONV_ERR_WORKSPACE;
    void *ws = nullptr;
    if ((st = noalloc_scratch(&ws)) != GCONV_OK) return st;
    const size_t part_bytes = ((size_t)p.N * p.gn_groups * p.slots * sizeof(float4) + 255) / 256 * 256;
    p.x = x; p.w = w; p.bias = bias; p.y = y; p.scale = scale;
    p.gn_part = reinterpret_cast<float4 *>(ws);
    if (launch_direct(p, tm, pl.geom, pl.KT, 1, pl.grid, pl.threads, pl.smem, stream) != cudaSuccess)
        return GCONV_ERR_CUDA;
    GnParams g;
    g.y = y;
    g.gn_part = p.gn_part;
    g.stats = reinterpret_cast<float2 *>(reinterpret_cast<char *>(ws) + part_bytes);
    g.gamma = gamma; g.beta = beta;
    g.N = s.N; g.K = s.K; g.gn_groups = gn_groups; g.kgn = s.K / gn_groups; g.slots = p.slots;
    g.PQ = (long long)s.P * s.Q;
    g.eps = eps;
    g.vec = (g.PQ % 4 == 0) && aligned16(y);
    const long long per_cta = g.vec ? 4LL * 256 * 8 : 256LL * 8;
    g.chunks = (int)((g.PQ + per_cta - 1) / per_cta);
    if (g.chunks < 1) g.chunks = 1;
    if (launch_gn_finalize(g, stream) != cudaSuccess) return GCONV_ERR_CUDA;
    if (launch_gn_normalize(g, stream) != cudaSuccess) return GCONV_ERR_CUDA;
    return GCONV_OK;
}

}  // extern "C"

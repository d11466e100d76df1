// Host-only replay of the planners' output (no GPU): the streaming direct
// kernel's stage layout, TMA box coordinates, thread-to-output mapping
// (every output written exactly once) and, on small shapes, its arithmetic on
// an emulated staged tile against a naive convolution; and the implicit GEMM's
// plans (shared memory, MMA N extent, tap-row folding, weight slices).
// Built and run by tests/test_host_planner.py; SWEEP_INC names the generated
// list of the 80 sweep shapes.
#include "gconv_api.cu"
#include <cstdio>
#include <vector>
#include <random>
struct GC { int R, S, ST, D, PAD; };
static GC geomc(int g) {
    switch (g) {
        case kGeom3x3s1p1: return {3,3,1,1,1};
        case kGeom3x3s1p0: return {3,3,1,1,0};
        case kGeom3x3s2p1: return {3,3,2,1,1};
        case kGeom5x9s1p0: return {5,9,1,1,0};
        case kGeom1x1s1p0: return {1,1,1,1,0};
    }
    return {0,0,0,0,0};
}
static int fails = 0;
#define CHECK(c, ...) do { if (!(c)) { if (fails < 20) { printf("FAIL %s:%d ", __FILE__, __LINE__); printf(__VA_ARGS__); printf("\n"); } ++fails; } } while (0)

static void check(int N, int C, int H, int W, int K, int R, int S, int st, int pad, int g, bool numerics,
                  int kt_req = 0) {
    Shape s;
    if (make_shape(s, N, C, H, W, K, R, S, st, pad, 1, g) != GCONV_OK) { printf("bad shape\n"); return; }
    int geom = match_geom(s);
    DirectPlan pl;
    if (!plan_stream(s, geom, true, pl, kt_req)) { printf("  %d %d %d %d %d %dx%d s%d p%d g%d: no stream plan\n", N,C,H,W,K,R,S,st,pad,g); return; }
    const DirectParams &p = pl.prm;
    GC gg = geomc(geom);
    const int HL = (gg.PAD + 3) / 4, OFF = 4 * HL - gg.PAD;
    const int WIN = OFF + 3 * gg.ST + (gg.S - 1) * gg.D + 1, NCH = (WIN + 3) / 4;
    const int KT = pl.KT, RPT = direct_rpt(KT), RS = gg.R * gg.S;
    const int IR = (RPT - 1) * gg.ST + (gg.R - 1) * gg.D + 1;
    CHECK(pl.smem == kStreamHeaderBytes + (size_t)p.stages * p.stage_floats * 4, "smem");
    CHECK(pl.smem <= 227 * 1024, "smem max %zu", pl.smem);
    CHECK(p.stages >= 1 && p.stages <= 8, "stages");
    CHECK(p.stage_floats % 32 == 0 && p.sw_off % 4 == 0 && p.pitch % 4 == 0, "alignment");
    CHECK(pl.threads % 32 == 0 && pl.threads <= 288 && pl.threads >= 64, "threads %d", pl.threads);
    CHECK(p.pitch <= 256 && p.IHt <= 256 && p.GB * p.cpg <= 256, "box");
    CHECK(p.CXP * p.RY * p.KZ * p.GB <= pl.threads - 32, "mapping fits");
    CHECK(p.KB == KT * p.KZ && p.KBtot == p.GB * p.KB && p.kpg % p.KB == 0, "channels");
    CHECK(p.pstride == p.IHt * p.pitch, "pstride");
    CHECK((long long)p.GB * p.cpg * p.pstride <= p.sw_off, "x region");
    CHECK(p.sw_off + p.cpg * RS * p.KBtot <= p.stage_floats, "w region");
    const int GY = p.n_kb * (p.groups / p.GB);
    CHECK((long long)N * GY * p.n_pt * p.n_qt == p.n_items, "items");
    const long long nout = (long long)N * K * s.P * s.Q;
    const bool cov = nout <= 40000000;
    std::vector<unsigned char> hit(cov ? nout : 0, 0);
    std::vector<float> x, w, y, yref;
    if (numerics) {
        std::mt19937 rng(N * 131 + C * 7 + H);
        std::uniform_real_distribution<float> U(-1.f, 1.f);
        x.resize((size_t)N * C * H * W); w.resize((size_t)K * s.cpg * RS); y.assign(nout, 0.f); yref.assign(nout, 0.f);
        for (auto &v : x) v = U(rng);
        for (auto &v : w) v = U(rng);
        for (int n = 0; n < N; ++n) for (int k = 0; k < K; ++k) for (int pp = 0; pp < s.P; ++pp) for (int q = 0; q < s.Q; ++q) {
            double a = 0; int gi = k / s.kpg;
            for (int c = 0; c < s.cpg; ++c) for (int r = 0; r < gg.R; ++r) for (int ss = 0; ss < gg.S; ++ss) {
                int ih = pp * gg.ST - gg.PAD + r, iw = q * gg.ST - gg.PAD + ss;
                if (ih < 0 || ih >= H || iw < 0 || iw >= W) continue;
                a += (double)w[((size_t)k * s.cpg + c) * RS + r * gg.S + ss] * x[(((size_t)n * C + gi * s.cpg + c) * H + ih) * W + iw];
            }
            yref[(((size_t)n * K + k) * s.P + pp) * s.Q + q] = (float)a;
        }
    }
    std::vector<float> stage(p.stage_floats);
    const int ncomp = pl.threads - 32;
    for (int it = 0; it < p.n_items; ++it) {
        int t = it;
        const int qt = t % p.n_qt; t /= p.n_qt;
        const int pt = t % p.n_pt; t /= p.n_pt;
        const int gy = t % GY; const int n = t / GY;
        const int g0 = (gy / p.n_kb) * p.GB;
        const int kc0 = g0 * p.kpg + (gy % p.n_kb) * p.KB;
        const int x0 = qt * p.TQ * gg.ST - 4 * HL, y0 = pt * p.TP * gg.ST - gg.PAD, z0 = n * p.C + g0 * p.cpg;
        CHECK(((x0 % 4) + 4) % 4 == 0, "tma x coordinate alignment %d", x0);
        CHECK(z0 + p.GB * p.cpg <= (n + 1) * p.C, "planes leave the image");
        CHECK(kc0 + p.KBtot <= K, "channels beyond K");
        if (numerics) {
            // TMA box emulation: [planes][IHt][pitch], zero fill outside
            for (int pl2 = 0; pl2 < p.GB * p.cpg; ++pl2) for (int r = 0; r < p.IHt; ++r) for (int c = 0; c < p.pitch; ++c) {
                int zi = z0 + pl2, yi = y0 + r, xi = x0 + c;
                float v = 0.f;
                if (yi >= 0 && yi < H && xi >= 0 && xi < W && zi < N * C) v = x[((size_t)zi * H + yi) * W + xi];
                stage[(size_t)pl2 * p.pstride + r * p.pitch + c] = v;
            }
            int nw = p.cpg * RS * p.KBtot;
            for (int e = 0; e < nw; ++e) {
                int kl = e % p.KBtot, crs = e / p.KBtot, c = crs / RS;
                stage[p.sw_off + e] = w[((size_t)(kc0 + kl) * p.cpg + c) * RS + (crs - c * RS)];
            }
        }
        for (int tid = 0; tid < ncomp; ++tid) {
            int u = tid;
            const int cx = u % p.CXP; u /= p.CXP;
            const int ry = u % p.RY; u /= p.RY;
            const int kz = u % p.KZ; const int gb = u / p.KZ;
            if (!(cx < p.CX && gb < p.GB)) continue;
            const int kl0 = gb * p.KB + kz * KT;
            std::vector<float> acc(RPT * 4 * KT, 0.f);
            for (int c = 0; c < p.cpg; ++c) {
                const long long xs = (long long)(gb * p.cpg + c) * p.pstride + (ry * RPT * gg.ST) * p.pitch + cx * gg.ST * 4;
                CHECK(xs % 4 == 0, "xs alignment");
                CHECK(xs + (IR - 1) * p.pitch + NCH * 4 <= (long long)(gb * p.cpg + c + 1) * p.pstride, "x read beyond plane (item %d tid %d)", it, tid);
                CHECK(cx * gg.ST * 4 + NCH * 4 <= p.pitch, "x read beyond row");
                const int ws = c * RS * p.KBtot + kl0;
                CHECK(ws + (RS - 1) * p.KBtot + KT <= p.cpg * RS * p.KBtot, "w read");
                if (numerics)
                    for (int r = 0; r < gg.R; ++r) for (int ss = 0; ss < gg.S; ++ss) for (int rp = 0; rp < RPT; ++rp) for (int v = 0; v < 4; ++v) {
                        float xv = stage[xs + (rp * gg.ST + r * gg.D) * p.pitch + OFF + v * gg.ST + ss * gg.D];
                        for (int k = 0; k < KT; ++k) acc[(rp * 4 + v) * KT + k] += stage[p.sw_off + ws + (r * gg.S + ss) * p.KBtot + k] * xv;
                    }
            }
            const int prow = pt * p.TP + ry * RPT, qb = qt * p.TQ + cx * 4;
            for (int rp = 0; rp < RPT; ++rp) {
                int pp = prow + rp; if (pp >= s.P) continue;
                for (int k = 0; k < KT; ++k) for (int v = 0; v < 4; ++v) {
                    int q = qb + v; if (q >= s.Q) continue;
                    long long o = (((long long)n * K + kc0 + kl0 + k) * s.P + pp) * s.Q + q;
                    if (cov) { CHECK(hit[o] == 0, "output written twice"); hit[o]++; }
                    if (numerics) y[o] = acc[(rp * 4 + v) * KT + k];
                }
            }
        }
    }
    if (cov) { long long miss = 0; for (auto h : hit) miss += h == 0; CHECK(miss == 0, "%lld outputs never written", miss); }
    if (numerics) {
        double md = 0; for (long long o = 0; o < nout; ++o) md = std::max(md, (double)fabs(y[o] - yref[o]));
        CHECK(md < 1e-4, "numerics max diff %g", md);
    }
    printf("  %3d %3d %3d %3d %3d %dx%d s%d p%d g%-3d: KT=%d CX=%d CXP=%d RY=%d KZ=%d GB=%d items=%d S=%d stage=%dB thr=%d smem=%zu %s\n",
           N, C, H, W, K, R, S, st, pad, g, KT, p.CX, p.CXP, p.RY, p.KZ, p.GB, p.n_items, p.stages, p.stage_floats * 4, pl.threads, pl.smem, numerics ? "num" : "");
}

int main() {
    // page workloads + test geometries that take the streaming path
    check(4, 144, 56, 56, 144, 3, 3, 1, 1, 144, true);
    check(1, 8, 16, 16, 8, 3, 3, 1, 1, 4, true);
    check(1, 32, 28, 28, 32, 3, 3, 1, 1, 8, true);
    check(2, 8, 33, 132, 8, 3, 3, 1, 1, 8, true);
    check(1, 16, 56, 56, 32, 3, 3, 1, 1, 16, true);
    check(2, 24, 20, 20, 48, 3, 3, 1, 1, 3, true);
    check(2, 16, 56, 56, 16, 3, 3, 2, 1, 16, true);
    check(1, 8, 32, 36, 8, 3, 3, 2, 1, 8, true);
    check(1, 8, 20, 24, 16, 3, 3, 1, 0, 1, true);
    check(1, 16, 12, 40, 16, 1, 1, 1, 0, 4, true);
    check(1, 96, 8, 12, 12, 5, 9, 1, 0, 1, true);
    check(1, 64, 12, 12, 64, 3, 3, 1, 1, 1, true);
    check(3, 12, 17, 24, 12, 3, 3, 1, 1, 12, true);
    check(2, 8, 300, 520, 8, 3, 3, 1, 1, 8, false);
    check(1, 8, 64, 1028, 8, 3, 3, 2, 1, 8, true);
    // the 80-shape sweep
    int shapes[80][4] = {
#include SWEEP_INC
    };
    for (int i = 0; i < 80; ++i) {
        int N = shapes[i][0], C = shapes[i][1], cpg = shapes[i][2], H = shapes[i][3];
        // every channels-per-thread choice the dispatch table can force
        for (int kt : {0, 1, 2, 4, 8})
            if (kt == 0 || cpg % kt == 0)
                check(N, C, H, H, C, 3, 3, 1, 1, C / cpg, kt == 0 && (long long)N * C * H * H * 9 * cpg < 3e7, kt);
    }
    // implicit-GEMM plans
    struct IG { int N, C, H, W, K, R, S, pad, g; bool chain; int gn; };
    const IG igs[] = {
        {8, 32, 512, 512, 64, 5, 9, 0, 1, false, 0}, {128, 8, 256, 256, 32, 3, 3, 0, 1, true, 8},
        {8, 32, 56, 56, 32, 3, 3, 1, 1, false, 0},   {8, 64, 56, 56, 64, 3, 3, 1, 1, false, 0},
        {1, 8, 9, 18, 128, 3, 3, 1, 1, false, 0},    {1, 8, 6, 10, 256, 3, 3, 1, 1, false, 0},
        {1, 16, 15, 50, 32, 5, 3, 2, 1, false, 0},   {1, 16, 12, 30, 64, 4, 1, 0, 1, false, 0},
        {1, 8, 13, 40, 32, 2, 3, 0, 1, false, 0},    {4, 512, 112, 112, 512, 3, 3, 1, 64, false, 0},
        {1, 24, 11, 21, 32, 3, 5, 1, 1, false, 0},   {2, 32, 20, 24, 64, 7, 7, 3, 1, false, 0},
        {8, 256, 28, 28, 256, 3, 3, 1, 8, false, 0}, {2, 8, 40, 44, 32, 3, 3, 0, 1, true, 8},
    };
    for (const IG &c : igs) {
        Shape s;
        CHECK(make_shape(s, c.N, c.C, c.H, c.W, c.K, c.R, c.S, 1, c.pad, 1, c.g) == GCONV_OK, "igemm shape");
        IgemmPlan pl;
        const int gp = igemm_pack(s);
        const Shape sp = gp ? packed_shape(s, gp) : s;
        if (!plan_igemm(sp, c.chain, c.gn, pl, false)) { CHECK(false, "no implicit-GEMM plan"); continue; }
        const IgemmParams &p = pl.prm;
        const int slices = p.CC8 * p.RC * (p.bs ? p.S : 1);
        CHECK(pl.smem <= 227 * 1024, "igemm smem %zu", pl.smem);
        CHECK(p.RF >= 1 && p.RF * p.RC >= p.R && (p.RF == 1 || p.RF * p.kpg <= 256), "fold RF %d RC %d", p.RF, p.RC);
        CHECK(p.RF == 1 || p.dil == 1, "fold needs dilation 1");
        CHECK(p.bs == 0 || p.RF > 1, "per-column slices without folding");
        CHECK(p.sa >= 1 && p.sa <= 4 && p.sb >= 1 && p.sb <= 4, "ring slots");
        CHECK(p.b_resident == (slices <= p.sb ? 1 : 0), "weight residency");
        CHECK(p.AR == p.TH + (p.R - 1) * p.dil, "staged rows");
        CHECK(2 * p.TH * p.kpg <= p.tmem_cols && p.tmem_cols <= 512, "tmem columns");
        if (c.chain && c.N == 128)   // the chain workload's measured plan: 3 tap rows folded, 7-row tiles
            CHECK(p.RF == 3 && p.TH == 7 && p.sa == 2, "chain plan RF %d TH %d sa %d", p.RF, p.TH, p.sa);
        printf("  igemm %3d %3d %4d %4d %3d %dx%d g%-3d chain%d: NT=%d TH=%d RF=%d RC=%d bs=%d sa=%d sb=%d smem=%zu\n",
               c.N, c.C, c.H, c.W, c.K, c.R, c.S, c.g, c.chain ? 1 : 0, p.kpg, p.TH, p.RF, p.RC, p.bs, p.sa, p.sb,
               pl.smem);
    }
    printf("%s (%d failures)\n", fails ? "FAILED" : "ALL OK", fails);
    return fails ? 1 : 0;
}

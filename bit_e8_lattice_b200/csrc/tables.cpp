// Host construction of the E8 core tables (see tables.h).
#include "tables.h"

#include <algorithm>
#include <array>
#include <mutex>

namespace e8q {
namespace {

struct Point {
    int n2;
    std::array<int8_t, 8> c;
};

int digit_of(int v) { return (v + 6) >> 1; }

int key4(const int8_t* c) {
    int k = 0;
    for (int i = 0; i < 4; ++i) k = k * 7 + digit_of(c[i]);
    return k;
}

bool build(HostTables& t) {
    // Every doubled E8 point with |P|^2 <= 48 (|p|^2 <= 12).  Even type:
    // coordinates in {-6,...,6} step 2; odd type: {-5,...,5} step 2.
    std::vector<Point> pts;
    pts.reserve(120000);
    for (int type = 0; type < 2; ++type) {
        const int nv = type ? 6 : 7;
        int dig[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        while (true) {
            Point p;
            int s = 0;
            p.n2 = 0;
            for (int i = 0; i < 8; ++i) {
                int v = 2 * dig[i] - 6 + type;
                p.c[i] = static_cast<int8_t>(v);
                s += v;
                p.n2 += v * v;
            }
            if (p.n2 <= 48 && ((s % 4) + 4) % 4 == 0) pts.push_back(p);
            int i = 7;
            for (; i >= 0; --i) {
                if (++dig[i] < nv) break;
                dig[i] = 0;
            }
            if (i < 0) break;
        }
    }
    std::sort(pts.begin(), pts.end(), [](const Point& a, const Point& b) {
        if (a.n2 != b.n2) return a.n2 < b.n2;
        return a.c < b.c;  // lexicographic on signed coordinates
    });
    if (pts.size() < static_cast<size_t>(kCoreSize)) return false;

    t.core.assign(static_cast<size_t>(kCoreSize) * 8, 0);
    for (int k = 0; k < kCoreSize; ++k)
        for (int i = 0; i < 8; ++i) t.core[8 * k + i] = pts[k].c[i];
    t.roots.clear();
    for (const Point& p : pts)
        if (p.n2 == 8)
            for (int i = 0; i < 8; ++i) t.roots.push_back(p.c[i]);
    if (t.roots.size() != static_cast<size_t>(kNumRoots) * 8) return false;
    t.root_of_key.assign(512, 0xFF);
    for (int k = 0; k < kNumRoots; ++k) {
        const int8_t* r = &t.roots[8 * k];
        int key = 0, nz = 0, first = -1, second = -1;
        for (int i = 0; i < 8; ++i)
            if (r[i] != 0) {
                ++nz;
                if (first < 0) first = i;
                else second = i;
            }
        if (nz == 2) {
            key = (first << 5) | (second << 2) | ((r[first] < 0) << 1) | (r[second] < 0);
        } else if (nz == 8) {
            key = 256;
            for (int i = 0; i < 8; ++i) key |= (r[i] < 0) << i;
        } else {
            return false;
        }
        if (t.root_of_key[key] != 0xFF) return false;
        t.root_of_key[key] = static_cast<uint8_t>(k);
    }

    // T2: position of a 4-vector among same-type 4-vectors with equal norm
    // and equal sum mod 4, in lexicographic order (= increasing key).
    t.t2.assign(kT2Size, 0xFFFF);
    for (int type = 0; type < 2; ++type) {
        std::vector<int> seen(49 * 4, 0);
        for (int key = 0; key < kKeySpace; ++key) {
            int d[4] = {key / 343, (key / 49) % 7, (key / 7) % 7, key % 7};
            int n2 = 0, s = 0;
            bool valid = true;
            for (int i = 0; i < 4; ++i) {
                if (type && d[i] > 5) valid = false;
                int v = 2 * d[i] - 6 + type;
                n2 += v * v;
                s += v;
            }
            if (!valid || n2 > 48) continue;
            int cls = n2 * 4 + ((s % 4) + 4) % 4;
            t.t2[type * kKeySpace + key] = static_cast<uint16_t>(seen[cls]++);
        }
    }

    // T1 = rank - T2, which must be the same for every point sharing
    // (type, head, |P|^2).
    std::vector<int32_t> t1(kT1Size, -1);
    for (size_t k = 0; k < pts.size(); ++k) {
        const Point& p = pts[k];
        int type = p.c[0] & 1;
        int hk = key4(p.c.data()), lk = key4(p.c.data() + 4);
        uint16_t t2v = t.t2[type * kKeySpace + lk];
        if (t2v == 0xFFFF) return false;
        int32_t val = static_cast<int32_t>(k) - t2v;
        int32_t& slot = t1[(type * kKeySpace + hk) * kNormLevels + p.n2 / 8];
        if (slot == -1) slot = val;
        else if (slot != val) return false;  // decomposition broken
    }
    t.t1.assign(kT1Size, 0xFFFF);
    for (int i = 0; i < kT1Size; ++i)
        if (t1[i] >= 0) t.t1[i] = static_cast<uint16_t>(std::min(t1[i], 0xFFFF));
    // every core point must be recognised by the saturated table
    for (int k = 0; k < kCoreSize; ++k) {
        const Point& p = pts[k];
        int type = p.c[0] & 1;
        uint16_t a = t.t1[(type * kKeySpace + key4(p.c.data())) * kNormLevels + p.n2 / 8];
        uint16_t b = t.t2[type * kKeySpace + key4(p.c.data() + 4)];
        if (a == 0xFFFF || a + b != k) return false;
    }
    // and no point past the core may look like a core point
    for (size_t k = kCoreSize; k < pts.size(); ++k) {
        const Point& p = pts[k];
        int type = p.c[0] & 1;
        uint16_t a = t.t1[(type * kKeySpace + key4(p.c.data())) * kNormLevels + p.n2 / 8];
        uint16_t b = t.t2[type * kKeySpace + key4(p.c.data() + 4)];
        if (a != 0xFFFF && a + b < kCoreSize) return false;
    }
    return true;
}

int ext_digit(int v) { return (v + 9) >> 1; }

int ext_key4(const int* c) {
    int k = 0;
    for (int i = 0; i < 4; ++i) k = k * 10 + ext_digit(c[i]);
    return k;
}

// The escape rule's root for P outside the core: largest <P, R>, ties to the
// lexicographically largest R.  Per coordinate a key (|P_i| << 5) | tie,
// tie = i for a negative coordinate and 23 - i otherwise: the two largest
// keys place the +-2 entries of the best integer-type root, the smallest
// key is the sign to flip for the half-type root when P has an odd number
// of negative coordinates.  Returns the construction key of the root
// (tables.h) and writes R.
int escape_root(const int (&P)[8], int (&R)[8]) {
    int k[8], sumw = 0;
    unsigned negm = 0;
    for (int i = 0; i < 8; ++i) {
        const bool neg = P[i] < 0;
        const int w = neg ? -P[i] : P[i];
        sumw += w;
        negm |= (neg ? 1u : 0u) << i;
        k[i] = (w << 5) | (neg ? i : 23 - i);
    }
    int m1 = k[0], mn = k[0];
    for (int i = 1; i < 8; ++i) {
        m1 = std::max(m1, k[i]);
        mn = std::min(mn, k[i]);
    }
    int m2 = 0;
    for (int i = 0; i < 8; ++i) m2 = std::max(m2, k[i] == m1 ? 0 : k[i]);
    auto pos_of = [](int tb) { return tb >= 16 ? 23 - tb : tb; };
    const int t1 = m1 & 31, t2 = m2 & 31, tn = mn & 31;
    const int p1 = pos_of(t1), p2 = pos_of(t2), pf = pos_of(tn);
    const int s1 = t1 >= 16 ? 2 : -2, s2 = t2 >= 16 ? 2 : -2;
    const int vI = 2 * ((m1 >> 5) + (m2 >> 5));
    const unsigned par = static_cast<unsigned>(__builtin_popcount(negm)) & 1u;
    const unsigned hneg = negm ^ (par << pf);
    const int vH = sumw - (par ? 2 * (mn >> 5) : 0);
    const int ri0 = p1 == 0 ? s1 : (p2 == 0 ? s2 : 0);
    const int rh0 = (hneg & 1u) ? -1 : 1;
    const bool useI = (vI > vH) || (vI == vH && ri0 > rh0);
    for (int i = 0; i < 8; ++i)
        R[i] = useI ? ((i == p1 ? s1 : 0) + (i == p2 ? s2 : 0)) : (((hneg >> i) & 1u) ? -1 : 1);
    if (useI) {
        const int lo = std::min(p1, p2), hi = std::max(p1, p2);
        const int nlo = (lo == p1 ? s1 : s2) < 0 ? 1 : 0, nhi = (hi == p1 ? s1 : s2) < 0 ? 1 : 0;
        return (lo << 5) | (hi << 2) | (nlo << 1) | nhi;
    }
    return 256 | static_cast<int>(hneg);
}

bool build_ext(HostTables& t) {
    // 4-vectors of each type with |v|^2 <= 88, grouped by (|v|^2, sum mod 4)
    struct Quad {
        int c[4];
        int n2, s4, key;
    };
    std::vector<Quad> quads[2];
    for (int type = 0; type < 2; ++type) {
        for (int a = -9; a <= 9; ++a)
            for (int b = -9; b <= 9; ++b)
                for (int c = -9; c <= 9; ++c)
                    for (int d = -9; d <= 9; ++d) {
                        const int v[4] = {a, b, c, d};
                        bool ok = true;
                        int n2 = 0, s = 0;
                        for (int i = 0; i < 4; ++i) {
                            if (((v[i] % 2) + 2) % 2 != type) ok = false;
                            n2 += v[i] * v[i];
                            s += v[i];
                        }
                        if (!ok || n2 > kExtMaxN2) continue;
                        Quad q;
                        for (int i = 0; i < 4; ++i) q.c[i] = v[i];
                        q.n2 = n2;
                        q.s4 = ((s % 4) + 4) % 4;
                        q.key = ext_key4(v);
                        quads[type].push_back(q);
                    }
    }
    // T2e: position of a tail among same-type tails of equal |t|^2 and sum mod 4,
    // lexicographic (= increasing key, digits are monotone in the coordinate)
    t.t2e.assign(kExtT2Size, kExtNone);
    for (int type = 0; type < 2; ++type) {
        std::vector<Quad> qs = quads[type];
        std::sort(qs.begin(), qs.end(), [](const Quad& x, const Quad& y) { return x.key < y.key; });
        std::vector<uint32_t> seen((kExtMaxN2 + 1) * 4, 0);
        for (const Quad& q : qs) t.t2e[type * kExtKeySpace + q.key] = seen[q.n2 * 4 + q.s4]++;
    }
    // every point: (|P|^2, lexicographic) order
    struct Pt {
        int n2;
        std::array<int8_t, 8> c;
    };
    std::vector<Pt> pts;
    pts.reserve(1200000);
    for (int type = 0; type < 2; ++type) {
        std::vector<std::vector<const Quad*>> bucket((kExtMaxN2 + 1) * 4);  // tails by (|t|^2, sum mod 4)
        for (const Quad& l : quads[type]) bucket[l.n2 * 4 + l.s4].push_back(&l);
        for (const Quad& h : quads[type])
            for (int n2t = 0; n2t + h.n2 <= kExtMaxN2; ++n2t)
                for (const Quad* lp : bucket[n2t * 4 + (4 - h.s4) % 4]) {
                const Quad& l = *lp;
                Pt p;
                p.n2 = h.n2 + l.n2;
                for (int i = 0; i < 4; ++i) {
                    p.c[i] = static_cast<int8_t>(h.c[i]);
                    p.c[4 + i] = static_cast<int8_t>(l.c[i]);
                }
                pts.push_back(p);
            }
    }
    std::sort(pts.begin(), pts.end(), [](const Pt& x, const Pt& y) {
        if (x.n2 != y.n2) return x.n2 < y.n2;
        return x.c < y.c;
    });
    if (pts.size() < static_cast<size_t>(kCoreSize)) return false;
    for (int k = 0; k < kCoreSize; ++k)  // the core comes first, in the same order
        for (int i = 0; i < 8; ++i)
            if (pts[k].c[i] != t.core[8 * k + i]) return false;
    // T1e = ext_rank - T2e, one value per (type, head, |P|^2 / 8)
    t.t1e.assign(kExtT1Size, kExtNone);
    for (size_t k = 0; k < pts.size(); ++k) {
        int c[8];
        for (int i = 0; i < 8; ++i) c[i] = pts[k].c[i];
        const int type = c[0] & 1;
        const uint32_t t2v = t.t2e[type * kExtKeySpace + ext_key4(c + 4)];
        if (t2v == kExtNone || t2v > k) return false;
        uint32_t& slot = t.t1e[(type * kExtKeySpace + ext_key4(c)) * kExtNormLevels + pts[k].n2 / 8];
        const uint32_t val = static_cast<uint32_t>(k) - t2v;
        if (slot == kExtNone) slot = val;
        else if (slot != val) return false;  // decomposition broken
    }
    // the encoding of every extended point
    t.res.assign(pts.size(), 0u);
    for (size_t k = 0; k < pts.size(); ++k) {
        if (k < static_cast<size_t>(kCoreSize)) {
            t.res[k] = static_cast<uint32_t>(k);
            continue;
        }
        int P[8], R[8], Q[8];
        for (int i = 0; i < 8; ++i) P[i] = pts[k].c[i];
        const int key = escape_root(P, R);
        for (int i = 0; i < 8; ++i) Q[i] = P[i] - R[i];
        const uint32_t rq = ext_rank(t, Q);
        const uint8_t root = t.root_of_key[key];
        if (rq != kExtNone && rq < static_cast<uint32_t>(kCoreSize) && root != 0xFF)
            t.res[k] = rq | (static_cast<uint32_t>(root) << 16) | (1u << 24);
        else
            t.res[k] = 2u << 24;
    }
    return true;
}

}  // namespace

uint32_t ext_rank(const HostTables& t, const int (&P)[8]) {
    int n2 = 0;
    for (int i = 0; i < 8; ++i) {
        if (P[i] < -9 || P[i] > 9) return kExtNone;
        n2 += P[i] * P[i];
    }
    if (n2 > kExtMaxN2) return kExtNone;
    const int type = P[0] & 1;
    const uint32_t a = t.t1e[(type * kExtKeySpace + ext_key4(P)) * kExtNormLevels + n2 / 8];
    const uint32_t b = t.t2e[type * kExtKeySpace + ext_key4(P + 4)];
    if (a == kExtNone || b == kExtNone) return kExtNone;
    return a + b;
}

const HostTables* host_tables() {
    static HostTables tables;
    static std::once_flag once;
    std::call_once(once, [] { tables.ok = build(tables) && build_ext(tables); });
    return tables.ok ? &tables : nullptr;
}

}  // namespace e8q

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

}  // namespace

const HostTables* host_tables() {
    static HostTables tables;
    static std::once_flag once;
    std::call_once(once, [] { tables.ok = build(tables); });
    return tables.ok ? &tables : nullptr;
}

}  // namespace e8q

// Dispatch table and cost model of the C ABI (include/spear_w4ec.h): the
// measured per-(M bucket, path, EC placement, EC on/off) times that
// spear_w4ec_tune records, exposed to a scheduler, and the tuned table saved
// to and loaded from JSON text.
//
// SPEAR, "A System for Post-Quantization Error-Adaptive Recovery Enabling
// Efficient Low-Bit LLM Serving", Abstract: an adaptive kernel-fusion dispatch
// keeps latency stable across configurations, and an SLO-constrained EC-aware
// scheduler keeps serving predictable.  The scheduler itself needs a serving
// system; what a kernel library can give it is the price of each choice.
#include <cctype>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>
#include <vector>

#include "handle.h"
#include "spear_w4ec.h"

using namespace spear;

namespace {

// Names of the eight cost slots (cost_index): path, placement, EC on/off.
const char *const kSlotNames[8] = {"decode+fused",      "decode+fused+ec_off", "decode+split",      "decode+split+ec_off",
                                   "tcgen05+fused",     "tcgen05+fused+ec_off", "tcgen05+split",     "tcgen05+split+ec_off"};

uint32_t flags_of_slot(int i)
{
    return ((i & 4) ? SPEAR_FORCE_TC : SPEAR_FORCE_DECODE) | ((i & 2) ? SPEAR_FORCE_SPLIT : SPEAR_FORCE_FUSED) |
           ((i & 1) ? SPEAR_EC_OFF : 0u);
}

int slot_of_name(const std::string &s)
{
    for (int i = 0; i < 8; ++i)
        if (s == kSlotNames[i])
            return i;
    return -1;
}

// ---- a small JSON reader: objects, arrays, strings (with \" and \\),
// numbers, true / false / null; enough for the table this file writes.
struct JValue {
    enum Kind { NUL, BOOL, NUM, STR, ARR, OBJ } kind = NUL;
    double num = 0.0;
    std::string str;
    std::vector<JValue> items;                          // ARR
    std::vector<std::pair<std::string, JValue>> members; // OBJ
    const JValue *get(const char *key) const
    {
        for (const auto &m : members)
            if (m.first == key)
                return &m.second;
        return nullptr;
    }
};

struct JReader {
    const char *p;
    int depth = 0;
    void ws()
    {
        while (*p && std::isspace((unsigned char)*p))
            ++p;
    }
    bool string(std::string &out)
    {
        if (*p != '"')
            return false;
        ++p;
        while (*p && *p != '"') {
            if (*p == '\\') {
                ++p;
                if (*p != '"' && *p != '\\' && *p != '/')
                    return false;
            }
            out.push_back(*p++);
        }
        if (*p != '"')
            return false;
        ++p;
        return true;
    }
    bool value(JValue &v)
    {
        if (++depth > 16)
            return false;
        ws();
        bool ok = false;
        if (*p == '{') {
            v.kind = JValue::OBJ;
            ++p;
            ws();
            if (*p == '}') {
                ++p;
                ok = true;
            } else {
                while (true) {
                    ws();
                    std::string key;
                    if (!string(key))
                        break;
                    ws();
                    if (*p != ':')
                        break;
                    ++p;
                    JValue item;
                    if (!value(item))
                        break;
                    v.members.emplace_back(key, std::move(item));
                    ws();
                    if (*p == ',') {
                        ++p;
                        continue;
                    }
                    if (*p == '}') {
                        ++p;
                        ok = true;
                    }
                    break;
                }
            }
        } else if (*p == '[') {
            v.kind = JValue::ARR;
            ++p;
            ws();
            if (*p == ']') {
                ++p;
                ok = true;
            } else {
                while (true) {
                    JValue item;
                    if (!value(item))
                        break;
                    v.items.push_back(std::move(item));
                    ws();
                    if (*p == ',') {
                        ++p;
                        continue;
                    }
                    if (*p == ']') {
                        ++p;
                        ok = true;
                    }
                    break;
                }
            }
        } else if (*p == '"') {
            v.kind = JValue::STR;
            ok = string(v.str);
        } else if (!std::strncmp(p, "true", 4) || !std::strncmp(p, "false", 5)) {
            v.kind = JValue::BOOL;
            v.num = *p == 't' ? 1.0 : 0.0;
            p += *p == 't' ? 4 : 5;
            ok = true;
        } else if (!std::strncmp(p, "null", 4)) {
            v.kind = JValue::NUL;
            p += 4;
            ok = true;
        } else {
            char *end = nullptr;
            v.num = std::strtod(p, &end);
            if (end != p) {
                v.kind = JValue::NUM;
                p = end;
                ok = true;
            }
        }
        --depth;
        return ok;
    }
};

bool as_int(const JValue *v, long long &out)
{
    if (!v || v->kind != JValue::NUM || v->num != (double)(long long)v->num)
        return false;
    out = (long long)v->num;
    return true;
}

std::string choice_name(uint32_t flags)
{
    std::string s = (flags & SPEAR_FORCE_TC) ? "tcgen05" : "decode";
    s += (flags & SPEAR_FORCE_SPLIT) ? "+split" : "+fused";
    return s;
}

int parse_choice(const std::string &s, uint32_t &flags)
{
    const int i = slot_of_name(s);
    if (i < 0 || (i & 1))
        return SPEAR_ERR_INVALID;   // a choice always carries the EC
    flags = flags_of_slot(i);
    return SPEAR_OK;
}

}  // namespace

extern "C" {

int spear_w4ec_cost(const spear_w4ec *h, int64_t M, uint32_t flags, float *us)
{
    if (!h || M <= 0 || !us)
        return SPEAR_ERR_INVALID;
    const uint32_t path = flags & (SPEAR_FORCE_DECODE | SPEAR_FORCE_TC);
    const uint32_t mode = flags & (SPEAR_FORCE_FUSED | SPEAR_FORCE_SPLIT);
    if ((path != SPEAR_FORCE_DECODE && path != SPEAR_FORCE_TC) ||
        (!(flags & SPEAR_EC_OFF) && mode != SPEAR_FORCE_FUSED && mode != SPEAR_FORCE_SPLIT) ||
        mode == (SPEAR_FORCE_FUSED | SPEAR_FORCE_SPLIT))
        return SPEAR_ERR_INVALID;
    const float c = h->cost_us[bucket_of(M)][cost_index(flags)];
    if (c < 0.0f)
        return SPEAR_ERR_STATE;
    *us = c;
    return SPEAR_OK;
}

int spear_w4ec_table_save(const spear_w4ec *h, char *buf, size_t cap, size_t *len)
{
    if (!h || !len)
        return SPEAR_ERR_INVALID;
    std::string out;
    char tmp[256];
    std::snprintf(tmp, sizeof tmp,
                  "{\"format\": \"spear_w4ec dispatch table\", \"version\": 1, \"K\": %lld, \"N\": %lld, \"r\": %d, "
                  "\"buckets\": [",
                  (long long)h->pk.K, (long long)h->pk.N, h->pk.r);
    out += tmp;
    bool first = true;
    for (int b = 0; b < 9; ++b) {
        bool any = h->table[b] != 0;
        for (float c : h->cost_us[b])
            any = any || c >= 0.0f;
        if (!any)
            continue;
        std::snprintf(tmp, sizeof tmp, "%s{\"bucket\": %d, \"M_max\": %lld, \"choice\": ", first ? "" : ", ", b,
                      b < 8 ? (long long)1 << b : -1LL);
        out += tmp;
        out += h->table[b] ? "\"" + choice_name(h->table[b]) + "\"" : std::string("null");
        out += ", \"us\": {";
        bool f2 = true;
        for (int i = 0; i < 8; ++i) {
            if (h->cost_us[b][i] < 0.0f)
                continue;
            std::snprintf(tmp, sizeof tmp, "%s\"%s\": %.9g", f2 ? "" : ", ", kSlotNames[i], (double)h->cost_us[b][i]);
            out += tmp;
            f2 = false;
        }
        out += "}}";
        first = false;
    }
    out += "]}";
    *len = out.size();
    if (!buf || cap < out.size() + 1)
        return SPEAR_ERR_INVALID;
    std::memcpy(buf, out.c_str(), out.size() + 1);
    return SPEAR_OK;
}

int spear_w4ec_table_load(spear_w4ec *h, const char *json)
{
    if (!h || !json)
        return SPEAR_ERR_INVALID;
    JReader rd{json};
    JValue root;
    if (!rd.value(root) || root.kind != JValue::OBJ)
        return SPEAR_ERR_INVALID;
    rd.ws();
    if (*rd.p)
        return SPEAR_ERR_INVALID;   // trailing text
    long long K = 0, N = 0, r = 0, version = 0;
    if (!as_int(root.get("version"), version) || version != 1 || !as_int(root.get("K"), K) ||
        !as_int(root.get("N"), N) || !as_int(root.get("r"), r))
        return SPEAR_ERR_INVALID;
    if (K != h->pk.K || N != h->pk.N || r != h->pk.r)
        return SPEAR_ERR_INVALID;   // a table of another layer shape
    const JValue *buckets = root.get("buckets");
    if (!buckets || buckets->kind != JValue::ARR)
        return SPEAR_ERR_INVALID;
    // check everything before changing the handle
    uint32_t table[9];
    float cost[9][8];
    std::memcpy(table, h->table, sizeof table);
    std::memcpy(cost, h->cost_us, sizeof cost);
    for (const JValue &bv : buckets->items) {
        long long b = -1;
        if (bv.kind != JValue::OBJ || !as_int(bv.get("bucket"), b) || b < 0 || b > 8)
            return SPEAR_ERR_INVALID;
        const JValue *ch = bv.get("choice");
        if (!ch)
            return SPEAR_ERR_INVALID;
        uint32_t flags = 0;
        if (ch->kind == JValue::STR) {
            if (parse_choice(ch->str, flags) != SPEAR_OK)
                return SPEAR_ERR_INVALID;
            if (!path_supported(h, flags & (SPEAR_FORCE_DECODE | SPEAR_FORCE_TC)))
                return SPEAR_ERR_UNSUPPORTED;
            if (h->pk.r == 0 && (flags & SPEAR_FORCE_SPLIT))
                return SPEAR_ERR_INVALID;
        } else if (ch->kind != JValue::NUL) {
            return SPEAR_ERR_INVALID;
        }
        table[b] = flags;
        const JValue *us = bv.get("us");
        if (us) {
            if (us->kind != JValue::OBJ)
                return SPEAR_ERR_INVALID;
            for (const auto &m : us->members) {
                const int i = slot_of_name(m.first);
                if (i < 0 || m.second.kind != JValue::NUM || !(m.second.num >= 0.0) || m.second.num > 1e9)
                    return SPEAR_ERR_INVALID;
                cost[b][i] = (float)m.second.num;
            }
        }
    }
    std::memcpy(h->table, table, sizeof table);
    std::memcpy(h->cost_us, cost, sizeof cost);
    return SPEAR_OK;
}

}  // extern "C"

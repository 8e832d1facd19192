// Selector artifact reader (host only).
//
// A selector artifact is a safetensors file: an 8-byte little-endian header
// length N, N bytes of a JSON object that maps each tensor name to its dtype,
// shape and [begin, end) byte range inside the data section, plus an optional
// "__metadata__" object of string pairs, then the data section.  The
// published competition artifact holds exactly 100 float16 tensors -- the
// query and key projections of 50 layers -- each of shape (56, 384, 128), in a
// file of at most 560,000,000 bytes, with metadata naming the miner's hotkey
// (tao.media, "Affine launches MiniMax-H3 video studio...", section "How the
// SN120 Competition Works").  The R2VA predictor is stored in FP8 and
// dequantised to BF16 at load (veyrul.com, "Veda R2VA for MiniMax-H3",
// second paragraph); no scale format is published, so FP8 (E4M3) tensors are
// read with a caller-given scale.
//
// The whole file is read once into memory; tensors are converted on request
// into a caller buffer (host) in fp32 or bf16.  Every byte range is checked
// against the file: ranges must lie inside the data section, match their
// dtype and shape exactly, and tile the data section without gaps or
// overlaps.  Parsing never trusts a length it has not checked.
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <cmath>
#include <map>
#include <string>
#include <vector>

#include "veda.h"

namespace {

enum class Dt { F16, BF16, F32, F8E4M3 };

struct TensorRec {
    std::string name;
    Dt dt;
    std::vector<int64_t> shape;
    uint64_t begin = 0, end = 0;   // inside the data section
};

// ---------------------------------------------------------------- JSON ---
// A small recursive-descent reader for the header: objects, arrays, strings
// (with escapes), integers; anything else in a header is a format error.
struct Json {
    enum Kind { OBJ, ARR, STR, NUM } kind = NUM;
    std::vector<std::pair<std::string, Json>> obj;
    std::vector<Json> arr;
    std::string str;
    int64_t num = 0;
};

struct Parser {
    const char* p;
    const char* e;
    int depth = 0;
    bool ok = true;

    void ws() { while (p < e && (*p == ' ' || *p == '\t' || *p == '\n' || *p == '\r')) ++p; }
    bool eat(char c)
    {
        ws();
        if (p < e && *p == c) { ++p; return true; }
        return false;
    }
    bool string(std::string& out)
    {
        ws();
        if (p >= e || *p != '"') return false;
        ++p;
        while (p < e && *p != '"') {
            char c = *p++;
            if (c == '\\') {
                if (p >= e) return false;
                const char x = *p++;
                switch (x) {
                case '"': case '\\': case '/': out += x; break;
                case 'b': out += '\b'; break;
                case 'f': out += '\f'; break;
                case 'n': out += '\n'; break;
                case 'r': out += '\r'; break;
                case 't': out += '\t'; break;
                case 'u': {
                    if (e - p < 4) return false;
                    unsigned v = 0;
                    for (int i = 0; i < 4; ++i) {
                        const char h = *p++;
                        v <<= 4;
                        if (h >= '0' && h <= '9') v |= (unsigned)(h - '0');
                        else if (h >= 'a' && h <= 'f') v |= (unsigned)(h - 'a' + 10);
                        else if (h >= 'A' && h <= 'F') v |= (unsigned)(h - 'A' + 10);
                        else return false;
                    }
                    if (v < 0x80) {
                        out += (char)v;
                    } else if (v < 0x800) {
                        out += (char)(0xC0 | (v >> 6));
                        out += (char)(0x80 | (v & 0x3F));
                    } else {   // surrogate halves are kept as three-byte sequences
                        out += (char)(0xE0 | (v >> 12));
                        out += (char)(0x80 | ((v >> 6) & 0x3F));
                        out += (char)(0x80 | (v & 0x3F));
                    }
                    break;
                }
                default: return false;
                }
            } else if ((unsigned char)c < 0x20) {
                return false;
            } else {
                out += c;
            }
        }
        if (p >= e) return false;
        ++p;   // closing quote
        return true;
    }
    bool value(Json& v)
    {
        if (++depth > 16) return false;
        ws();
        if (p >= e) return false;
        bool r;
        if (*p == '{') {
            ++p;
            v.kind = Json::OBJ;
            r = true;
            if (!eat('}')) {
                do {
                    std::string k;
                    Json x;
                    if (!string(k) || !eat(':') || !value(x)) { r = false; break; }
                    v.obj.emplace_back(std::move(k), std::move(x));
                } while (eat(','));
                if (r) r = eat('}');
            }
        } else if (*p == '[') {
            ++p;
            v.kind = Json::ARR;
            r = true;
            if (!eat(']')) {
                do {
                    Json x;
                    if (!value(x)) { r = false; break; }
                    v.arr.push_back(std::move(x));
                } while (eat(','));
                if (r) r = eat(']');
            }
        } else if (*p == '"') {
            v.kind = Json::STR;
            r = string(v.str);
        } else {
            // a non-negative integer (sizes and offsets); no fractions or exponents
            v.kind = Json::NUM;
            int64_t x = 0;
            int nd = 0;
            while (p < e && *p >= '0' && *p <= '9' && nd < 19) {
                x = x * 10 + (*p++ - '0');
                ++nd;
            }
            r = nd > 0 && !(p < e && (*p >= '0' && *p <= '9'));
            v.num = x;
        }
        --depth;
        return r;
    }
};

bool parse_dtype(const std::string& s, Dt* dt, int* size)
{
    if (s == "F16") { *dt = Dt::F16; *size = 2; return true; }
    if (s == "BF16") { *dt = Dt::BF16; *size = 2; return true; }
    if (s == "F32") { *dt = Dt::F32; *size = 4; return true; }
    if (s == "F8_E4M3") { *dt = Dt::F8E4M3; *size = 1; return true; }
    return false;
}

// ---------------------------------------------------------- conversions ---
float f32_bits(uint32_t u)
{
    float f;
    memcpy(&f, &u, 4);
    return f;
}

uint32_t bits_f32(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    return u;
}

// IEEE binary16 -> binary32 (exact): sign, 5-bit exponent (bias 15),
// 10-bit fraction; subnormals, infinities and NaN kept.
float half_to_float(uint16_t h)
{
    const uint32_t sign = (uint32_t)(h >> 15) << 31;
    const int exp = (h >> 10) & 0x1F;
    const uint32_t frac = h & 0x3FF;
    if (exp == 0x1F) return f32_bits(sign | 0x7F800000u | (frac << 13));   // inf / NaN
    if (exp == 0) {                                                       // zero / subnormal
        const float mag = std::ldexp((float)frac, -24);
        return sign ? -mag : mag;
    }
    return f32_bits(sign | ((uint32_t)(exp - 15 + 127) << 23) | (frac << 13));
}

// OCP FP8 E4M3 ("fn": no infinities; S.1111.111 is NaN) -> binary32 (exact):
// 4-bit exponent (bias 7), 3-bit fraction, subnormals.
float e4m3_to_float(uint8_t b)
{
    const bool neg = (b & 0x80) != 0;
    const int exp = (b >> 3) & 0xF;
    const int frac = b & 0x7;
    float mag;
    if (exp == 0xF && frac == 0x7) return std::nanf("");
    if (exp == 0) mag = std::ldexp((float)frac, -9);          // subnormal: frac/8 * 2^-6
    else mag = std::ldexp(1.0f + (float)frac / 8.0f, exp - 7);
    return neg ? -mag : mag;
}

// binary32 -> bfloat16, round to nearest, ties to even; NaN stays a (quiet) NaN.
uint16_t float_to_bf16(float f)
{
    const uint32_t u = bits_f32(f);
    if ((u & 0x7FFFFFFFu) > 0x7F800000u) return (uint16_t)((u >> 16) | 0x0040u);
    const uint32_t rounded = u + 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(rounded >> 16);
}

}  // namespace

struct veda_selector {
    std::vector<uint8_t> file;
    uint64_t data_off = 0;          // start of the data section in `file`
    std::vector<TensorRec> tensors; // in data order
    std::vector<std::pair<std::string, std::string>> meta;
};

extern "C" {

veda_status veda_selector_open(const char* path, veda_selector** out)
{
    if (!path || !out) return VEDA_ERR_INVALID_ARG;
    *out = nullptr;
    FILE* f = fopen(path, "rb");
    if (!f) return VEDA_ERR_IO;
    veda_selector* s = new veda_selector();
    bool io_ok = fseek(f, 0, SEEK_END) == 0;
    const long sz = io_ok ? ftell(f) : -1;
    io_ok = io_ok && sz >= 0 && fseek(f, 0, SEEK_SET) == 0;
    if (io_ok) {
        s->file.resize((size_t)sz);
        io_ok = sz == 0 || fread(s->file.data(), 1, (size_t)sz, f) == (size_t)sz;
    }
    fclose(f);
    if (!io_ok) {
        delete s;
        return VEDA_ERR_IO;
    }
    auto fail = [&]() {
        delete s;
        return VEDA_ERR_FORMAT;
    };
    const uint64_t total = s->file.size();
    if (total < 8) return fail();
    uint64_t hlen = 0;
    for (int i = 7; i >= 0; --i) hlen = (hlen << 8) | s->file[(size_t)i];
    if (hlen < 2 || hlen > total - 8 || hlen > (uint64_t)100 << 20) return fail();
    Parser ps{reinterpret_cast<const char*>(s->file.data()) + 8,
              reinterpret_cast<const char*>(s->file.data()) + 8 + hlen};
    Json root;
    if (!ps.value(root) || root.kind != Json::OBJ) return fail();
    ps.ws();
    if (ps.p != ps.e) return fail();   // trailing bytes in the header (spaces are allowed above)
    s->data_off = 8 + hlen;
    const uint64_t data_len = total - s->data_off;
    std::map<std::string, int> seen;
    for (auto& kv : root.obj) {
        if (seen.count(kv.first)) return fail();   // duplicate key
        seen[kv.first] = 1;
        if (kv.first == "__metadata__") {
            if (kv.second.kind != Json::OBJ) return fail();
            for (auto& m : kv.second.obj) {
                if (m.second.kind != Json::STR) return fail();
                s->meta.emplace_back(m.first, m.second.str);
            }
            continue;
        }
        const Json& t = kv.second;
        if (t.kind != Json::OBJ) return fail();
        const Json *jd = nullptr, *js = nullptr, *jo = nullptr;
        for (auto& f2 : t.obj) {
            if (f2.first == "dtype") jd = &f2.second;
            else if (f2.first == "shape") js = &f2.second;
            else if (f2.first == "data_offsets") jo = &f2.second;
            else return fail();
        }
        if (!jd || !js || !jo || jd->kind != Json::STR || js->kind != Json::ARR || jo->kind != Json::ARR ||
            jo->arr.size() != 2 || js->arr.size() > 8)
            return fail();
        TensorRec r;
        r.name = kv.first;
        int esz = 0;
        if (!parse_dtype(jd->str, &r.dt, &esz)) return fail();
        uint64_t count = 1;
        for (auto& d : js->arr) {
            if (d.kind != Json::NUM || d.num < 0 || d.num > ((int64_t)1 << 40)) return fail();
            r.shape.push_back(d.num);
            count *= (uint64_t)d.num;
            if (count > ((uint64_t)1 << 40)) return fail();
        }
        if (jo->arr[0].kind != Json::NUM || jo->arr[1].kind != Json::NUM) return fail();
        r.begin = (uint64_t)jo->arr[0].num;
        r.end = (uint64_t)jo->arr[1].num;
        if (r.begin > r.end || r.end > data_len || r.end - r.begin != count * (uint64_t)esz) return fail();
        s->tensors.push_back(std::move(r));
    }
    // the byte ranges tile the data section exactly
    std::sort(s->tensors.begin(), s->tensors.end(),
              [](const TensorRec& a, const TensorRec& b) { return a.begin < b.begin; });
    uint64_t at = 0;
    for (auto& r : s->tensors) {
        if (r.begin != at) return fail();
        at = r.end;
    }
    if (at != data_len) return fail();
    *out = s;
    return VEDA_OK;
}

void veda_selector_close(veda_selector* s) { delete s; }

veda_status veda_selector_check(const veda_selector* s, int32_t n_tensors, const int64_t* shape, int32_t ndim,
                                int64_t max_file_bytes, const char* required_meta_key)
{
    if (!s || n_tensors < 0 || ndim < 0 || ndim > 8 || (ndim > 0 && !shape)) return VEDA_ERR_INVALID_ARG;
    if ((int64_t)s->tensors.size() != n_tensors) return VEDA_ERR_FORMAT;
    if (max_file_bytes > 0 && (int64_t)s->file.size() > max_file_bytes) return VEDA_ERR_FORMAT;
    for (auto& r : s->tensors) {
        if (r.dt != Dt::F16 && r.dt != Dt::F8E4M3) return VEDA_ERR_FORMAT;
        if ((int32_t)r.shape.size() != ndim) return VEDA_ERR_FORMAT;
        for (int i = 0; i < ndim; ++i)
            if (r.shape[(size_t)i] != shape[i]) return VEDA_ERR_FORMAT;
    }
    if (required_meta_key) {
        bool found = false;
        for (auto& m : s->meta) found = found || (m.first == required_meta_key && !m.second.empty());
        if (!found) return VEDA_ERR_FORMAT;
    }
    return VEDA_OK;
}

int32_t veda_selector_count(const veda_selector* s) { return s ? (int32_t)s->tensors.size() : -1; }

veda_status veda_selector_find(const veda_selector* s, const char* name, int32_t* index)
{
    if (!s || !name || !index) return VEDA_ERR_INVALID_ARG;
    for (size_t i = 0; i < s->tensors.size(); ++i)
        if (s->tensors[i].name == name) {
            *index = (int32_t)i;
            return VEDA_OK;
        }
    return VEDA_ERR_INVALID_ARG;
}

veda_status veda_selector_info(const veda_selector* s, int32_t i, const char** name, const char** dtype,
                               int32_t* ndim, int64_t* shape)
{
    if (!s || i < 0 || (size_t)i >= s->tensors.size()) return VEDA_ERR_INVALID_ARG;
    const TensorRec& r = s->tensors[(size_t)i];
    static const char* names[] = {"F16", "BF16", "F32", "F8_E4M3"};
    if (name) *name = r.name.c_str();
    if (dtype) *dtype = names[(int)r.dt];
    if (ndim) *ndim = (int32_t)r.shape.size();
    if (shape)
        for (size_t k = 0; k < r.shape.size(); ++k) shape[k] = r.shape[k];
    return VEDA_OK;
}

const char* veda_selector_metadata(const veda_selector* s, const char* key)
{
    if (!s || !key) return nullptr;
    for (auto& m : s->meta)
        if (m.first == key) return m.second.c_str();
    return nullptr;
}

veda_status veda_selector_read(const veda_selector* s, int32_t i, veda_dtype out_dtype, float scale, void* dst,
                               size_t dst_bytes)
{
    if (!s || i < 0 || (size_t)i >= s->tensors.size() || !dst) return VEDA_ERR_INVALID_ARG;
    if (out_dtype != VEDA_F32 && out_dtype != VEDA_BF16) return VEDA_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !std::isfinite(scale)) return VEDA_ERR_INVALID_ARG;
    const TensorRec& r = s->tensors[(size_t)i];
    const int esz = r.dt == Dt::F32 ? 4 : r.dt == Dt::F8E4M3 ? 1 : 2;
    const uint64_t count = (r.end - r.begin) / (uint64_t)esz;
    const size_t osz = out_dtype == VEDA_F32 ? 4 : 2;
    if (dst_bytes < count * osz) return VEDA_ERR_INVALID_ARG;
    const uint8_t* src = s->file.data() + s->data_off + r.begin;
    for (uint64_t k = 0; k < count; ++k) {
        float v;
        switch (r.dt) {
        case Dt::F16: v = half_to_float((uint16_t)(src[2 * k] | (src[2 * k + 1] << 8))); break;
        case Dt::BF16: v = f32_bits((uint32_t)(src[2 * k] | (src[2 * k + 1] << 8)) << 16); break;
        case Dt::F32: {
            uint32_t u = (uint32_t)src[4 * k] | ((uint32_t)src[4 * k + 1] << 8) | ((uint32_t)src[4 * k + 2] << 16) |
                         ((uint32_t)src[4 * k + 3] << 24);
            v = f32_bits(u);
            break;
        }
        default: v = e4m3_to_float(src[k]); break;
        }
        if (scale != 1.f) v *= scale;
        if (out_dtype == VEDA_F32) static_cast<float*>(dst)[k] = v;
        else static_cast<uint16_t*>(dst)[k] = float_to_bf16(v);
    }
    return VEDA_OK;
}

}  // extern "C"

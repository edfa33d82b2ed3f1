// C ABI of the library (include/mlxq.h): argument validation, the
// safetensors reader behind mlxq_load ("MlxInt8Weight" page, load), buffer
// ownership (release) and kernel selection.  No computation happens here; every
// step of the layer runs in the CUDA kernels.
#include <cuda_runtime.h>

#include <atomic>
#include <cerrno>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/mlxq.h"
#include "kernels.h"

namespace mlxq {

// The library's device status word (see mlxq_device_status).  Kernels get its
// address as an argument.
__device__ unsigned int g_status_word;

namespace {

thread_local std::string g_err;

int fail(int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_err = buf;
    return code;
}

int ok() { return MLXQ_OK; }

constexpr int kMaxDevices = 64;
std::mutex g_dev_mu;
DeviceInfo g_dev[kMaxDevices];
std::atomic<bool> g_dev_ready[kMaxDevices];
unsigned int* g_status_ptr[kMaxDevices];

// ---- minimal JSON reader for the safetensors header ---------------------------------
struct JVal {
    enum Kind { NUL, BOOL, NUM, STR, ARR, OBJ } kind = NUL;
    bool b = false;
    double num = 0;
    bool is_int = false;
    long long i = 0;
    std::string s;
    std::vector<JVal> arr;
    std::vector<std::pair<std::string, JVal>> obj;
    const JVal* get(const std::string& k) const {
        for (const auto& kv : obj)
            if (kv.first == k) return &kv.second;
        return nullptr;
    }
};

struct JParser {
    const char* p;
    const char* e;
    int depth = 0;
    bool err = false;

    void ws() {
        while (p < e && (*p == ' ' || *p == '\t' || *p == '\n' || *p == '\r')) ++p;
    }
    bool lit(const char* t) {
        size_t n = strlen(t);
        if (static_cast<size_t>(e - p) < n || memcmp(p, t, n) != 0) return false;
        p += n;
        return true;
    }
    static void put_utf8(std::string& o, unsigned cp) {
        if (cp < 0x80) {
            o += static_cast<char>(cp);
        } else if (cp < 0x800) {
            o += static_cast<char>(0xC0 | (cp >> 6));
            o += static_cast<char>(0x80 | (cp & 0x3F));
        } else if (cp < 0x10000) {
            o += static_cast<char>(0xE0 | (cp >> 12));
            o += static_cast<char>(0x80 | ((cp >> 6) & 0x3F));
            o += static_cast<char>(0x80 | (cp & 0x3F));
        } else {
            o += static_cast<char>(0xF0 | (cp >> 18));
            o += static_cast<char>(0x80 | ((cp >> 12) & 0x3F));
            o += static_cast<char>(0x80 | ((cp >> 6) & 0x3F));
            o += static_cast<char>(0x80 | (cp & 0x3F));
        }
    }
    bool hex4(unsigned& v) {
        if (e - p < 4) return false;
        v = 0;
        for (int i = 0; i < 4; ++i) {
            char c = *p++;
            v <<= 4;
            if (c >= '0' && c <= '9') v |= c - '0';
            else if (c >= 'a' && c <= 'f') v |= c - 'a' + 10;
            else if (c >= 'A' && c <= 'F') v |= c - 'A' + 10;
            else return false;
        }
        return true;
    }
    bool str(std::string& o) {
        if (p >= e || *p != '"') return false;
        ++p;
        while (p < e && *p != '"') {
            unsigned char c = static_cast<unsigned char>(*p);
            if (c < 0x20) return false;
            if (c != '\\') {
                o += static_cast<char>(c);
                ++p;
                continue;
            }
            if (++p >= e) return false;
            char q = *p++;
            switch (q) {
                case '"': o += '"'; break;
                case '\\': o += '\\'; break;
                case '/': o += '/'; break;
                case 'b': o += '\b'; break;
                case 'f': o += '\f'; break;
                case 'n': o += '\n'; break;
                case 'r': o += '\r'; break;
                case 't': o += '\t'; break;
                case 'u': {
                    unsigned cp;
                    if (!hex4(cp)) return false;
                    if (cp >= 0xD800 && cp < 0xDC00) {
                        unsigned lo;
                        if (e - p < 6 || p[0] != '\\' || p[1] != 'u') return false;
                        p += 2;
                        if (!hex4(lo) || lo < 0xDC00 || lo >= 0xE000) return false;
                        cp = 0x10000 + ((cp - 0xD800) << 10) + (lo - 0xDC00);
                    }
                    put_utf8(o, cp);
                    break;
                }
                default: return false;
            }
        }
        if (p >= e) return false;
        ++p;
        return true;
    }
    bool num(JVal& v) {
        const char* s = p;
        if (p < e && *p == '-') ++p;
        if (p >= e || *p < '0' || *p > '9') return false;
        bool integral = true;
        while (p < e && ((*p >= '0' && *p <= '9') || *p == '.' || *p == 'e' || *p == 'E' ||
                         *p == '+' || *p == '-')) {
            if (*p == '.' || *p == 'e' || *p == 'E') integral = false;
            ++p;
        }
        std::string t(s, p);
        char* endp = nullptr;
        v.kind = JVal::NUM;
        v.num = strtod(t.c_str(), &endp);
        if (endp != t.c_str() + t.size()) return false;
        v.is_int = false;
        if (integral) {
            errno = 0;
            long long iv = strtoll(t.c_str(), &endp, 10);
            if (errno == 0 && endp == t.c_str() + t.size()) {
                v.is_int = true;
                v.i = iv;
            }
        }
        return true;
    }
    bool value(JVal& v) {
        if (++depth > 64) return false;
        ws();
        if (p >= e) return false;
        bool r = false;
        if (*p == '{') {
            ++p;
            v.kind = JVal::OBJ;
            ws();
            if (p < e && *p == '}') {
                ++p;
                r = true;
            } else {
                for (;;) {
                    ws();
                    std::string k;
                    if (!str(k)) break;
                    ws();
                    if (p >= e || *p != ':') break;
                    ++p;
                    JVal c;
                    if (!value(c)) break;
                    v.obj.emplace_back(std::move(k), std::move(c));
                    ws();
                    if (p < e && *p == ',') {
                        ++p;
                        continue;
                    }
                    if (p < e && *p == '}') {
                        ++p;
                        r = true;
                    }
                    break;
                }
            }
        } else if (*p == '[') {
            ++p;
            v.kind = JVal::ARR;
            ws();
            if (p < e && *p == ']') {
                ++p;
                r = true;
            } else {
                for (;;) {
                    JVal c;
                    if (!value(c)) break;
                    v.arr.push_back(std::move(c));
                    ws();
                    if (p < e && *p == ',') {
                        ++p;
                        continue;
                    }
                    if (p < e && *p == ']') {
                        ++p;
                        r = true;
                    }
                    break;
                }
            }
        } else if (*p == '"') {
            v.kind = JVal::STR;
            r = str(v.s);
        } else if (lit("true")) {
            v.kind = JVal::BOOL;
            v.b = true;
            r = true;
        } else if (lit("false")) {
            v.kind = JVal::BOOL;
            r = true;
        } else if (lit("null")) {
            v.kind = JVal::NUL;
            r = true;
        } else {
            r = num(v);
        }
        --depth;
        return r;
    }
};

struct TensorInfo {
    std::string dtype;
    std::vector<long long> shape;
    size_t begin = 0, end = 0;
};

long long dtype_size(const std::string& d) {
    static const std::map<std::string, long long> sz = {
        {"BOOL", 1}, {"U8", 1}, {"I8", 1}, {"F8_E5M2", 1}, {"F8_E4M3", 1}, {"I16", 2},
        {"U16", 2},  {"F16", 2}, {"BF16", 2}, {"I32", 4},   {"U32", 4},     {"F32", 4},
        {"F64", 8},  {"I64", 8}, {"U64", 8}};
    auto it = sz.find(d);
    return it == sz.end() ? -1 : it->second;
}

// Parse the blob; on success fills `tensors` and `data` (start of the data
// section) and returns MLXQ_OK.
int parse_safetensors(const uint8_t* blob, size_t len, std::map<std::string, TensorInfo>& tensors,
                      const uint8_t*& data, size_t& data_len) {
    if (len < 8) return fail(MLXQ_ERR_PARSE, "safetensors blob shorter than its 8-byte header length");
    uint64_t hlen = 0;
    for (int i = 0; i < 8; ++i) hlen |= static_cast<uint64_t>(blob[i]) << (8 * i);
    if (hlen > len - 8) return fail(MLXQ_ERR_PARSE, "safetensors header length %llu exceeds the blob",
                                    static_cast<unsigned long long>(hlen));
    JParser jp{reinterpret_cast<const char*>(blob + 8), reinterpret_cast<const char*>(blob + 8 + hlen)};
    JVal root;
    if (!jp.value(root)) return fail(MLXQ_ERR_PARSE, "safetensors header is not valid JSON");
    jp.ws();
    if (jp.p != jp.e) return fail(MLXQ_ERR_PARSE, "trailing bytes after the safetensors JSON header");
    if (root.kind != JVal::OBJ) return fail(MLXQ_ERR_PARSE, "safetensors header is not a JSON object");
    data = blob + 8 + hlen;
    data_len = len - 8 - hlen;
    for (const auto& kv : root.obj) {
        if (kv.first == "__metadata__") continue;
        const JVal& t = kv.second;
        const JVal* dt = t.get("dtype");
        const JVal* sh = t.get("shape");
        const JVal* off = t.get("data_offsets");
        if (t.kind != JVal::OBJ || !dt || dt->kind != JVal::STR || !sh || sh->kind != JVal::ARR || !off ||
            off->kind != JVal::ARR || off->arr.size() != 2)
            return fail(MLXQ_ERR_PARSE, "tensor '%s': malformed entry", kv.first.c_str());
        TensorInfo ti;
        ti.dtype = dt->s;
        long long count = 1;
        for (const JVal& d : sh->arr) {
            if (d.kind != JVal::NUM || !d.is_int || d.i < 0)
                return fail(MLXQ_ERR_PARSE, "tensor '%s': bad dimension", kv.first.c_str());
            if (d.i != 0 && count > (1LL << 62) / d.i)
                return fail(MLXQ_ERR_PARSE, "tensor '%s': shape overflows", kv.first.c_str());
            count *= d.i;
            ti.shape.push_back(d.i);
        }
        const JVal& b0 = off->arr[0];
        const JVal& b1 = off->arr[1];
        if (b0.kind != JVal::NUM || b1.kind != JVal::NUM || !b0.is_int || !b1.is_int || b0.i < 0 ||
            b1.i < b0.i || static_cast<unsigned long long>(b1.i) > data_len)
            return fail(MLXQ_ERR_PARSE, "tensor '%s': data_offsets outside the data section",
                        kv.first.c_str());
        ti.begin = static_cast<size_t>(b0.i);
        ti.end = static_cast<size_t>(b1.i);
        const long long es = dtype_size(ti.dtype);
        if (es > 0 && static_cast<long long>(ti.end - ti.begin) != count * es)
            return fail(MLXQ_ERR_PARSE, "tensor '%s': byte size does not match its shape and dtype",
                        kv.first.c_str());
        tensors[kv.first] = std::move(ti);
    }
    return MLXQ_OK;
}

// ---- argument checks ------------------------------------------------------------------
bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int check_weight(const mlxq_weight* w, WeightView& v) {
    if (!w) return fail(MLXQ_ERR_INVALID_ARG, "null weight handle");
    if (!w->packed || !w->scales || !w->biases)
        return fail(MLXQ_ERR_INVALID_ARG, "weight handle is released or was never loaded");
    if (w->in_features % 4 != 0)
        return fail(MLXQ_ERR_SHAPE, "in_features %u is not a multiple of 4", w->in_features);
    if (w->group_size == 0 || w->in_features % w->group_size != 0)
        return fail(MLXQ_ERR_GROUP_SIZE, "group_size %u does not divide in_features %u", w->group_size,
                    w->in_features);
    if (!aligned(w->packed, 4) || !aligned(w->scales, 2) || !aligned(w->biases, 2))
        return fail(MLXQ_ERR_INVALID_ARG, "weight buffers are misaligned");
    // every byte count below (up to 4 bytes per weight, times m for gemm
    // outputs checked separately) must stay far inside int64
    if (static_cast<uint64_t>(w->out_features) * w->in_features > (1ull << 50))
        return fail(MLXQ_ERR_SHAPE, "out_features x in_features = %llu is beyond any device",
                    static_cast<unsigned long long>(static_cast<uint64_t>(w->out_features) * w->in_features));
    v.packed = static_cast<const uint32_t*>(w->packed);
    v.scales = static_cast<const uint16_t*>(w->scales);
    v.biases = static_cast<const uint16_t*>(w->biases);
    v.N = w->out_features;
    v.K = w->in_features;
    v.gs = w->group_size;
    v.G = v.K / v.gs;
    if (w->flags & ~MLXQ_WEIGHT_STATIC)
        return fail(MLXQ_ERR_INVALID_ARG, "unknown weight flags 0x%x", w->flags & ~MLXQ_WEIGHT_STATIC);
    v.flags = w->flags;
    return MLXQ_OK;
}

int check_buf(const void* p, int64_t elems, const char* name) {
    if (elems == 0) return MLXQ_OK;
    if (!p) return fail(MLXQ_ERR_INVALID_ARG, "%s is null", name);
    if (!aligned(p, 2)) return fail(MLXQ_ERR_INVALID_ARG, "%s is not 2-byte aligned", name);
    return MLXQ_OK;
}

bool overlap(const void* a, int64_t abytes, const void* b, int64_t bbytes) {
    if (!a || !b || abytes == 0 || bbytes == 0) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + static_cast<uintptr_t>(bbytes) && b0 < a0 + static_cast<uintptr_t>(abytes);
}

int check_out_vs_weight(const void* out, int64_t obytes, const WeightView& v) {
    if (overlap(out, obytes, v.packed, v.N * v.K) || overlap(out, obytes, v.scales, v.N * v.G * 2) ||
        overlap(out, obytes, v.biases, v.N * v.G * 2))
        return fail(MLXQ_ERR_INVALID_ARG, "output overlaps the weight buffers");
    return MLXQ_OK;
}

int launch_status(cudaError_t e, const char* what) {
    if (e != cudaSuccess) return fail(MLXQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    return MLXQ_OK;
}

cudaStream_t as_stream(uint64_t s) { return reinterpret_cast<cudaStream_t>(static_cast<uintptr_t>(s)); }

// mlxq_selftest_fail_alloc: the n-th device allocation of mlxq_load from now
// fails as if cudaMalloc had run out (0: none).
std::atomic<int> g_fail_alloc_in{0};
bool take_injected_alloc_failure() {
    int n = g_fail_alloc_in.load();
    while (n > 0) {
        if (g_fail_alloc_in.compare_exchange_weak(n, n - 1)) return n == 1;
    }
    return false;
}

}  // namespace

const DeviceInfo& device_info() {
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= kMaxDevices) dev = 0;
    if (g_dev_ready[dev].load(std::memory_order_acquire)) return g_dev[dev];
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (!g_dev_ready[dev].load(std::memory_order_relaxed)) {
        DeviceInfo di{};
        di.device = dev;
        cudaDeviceGetAttribute(&di.sm_count, cudaDevAttrMultiProcessorCount, dev);
        cudaDeviceGetAttribute(&di.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        cudaDeviceGetAttribute(&di.smem_per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
        if (di.sm_count <= 0) di.sm_count = 1;
        if (di.max_smem_optin <= 0) di.max_smem_optin = 48 * 1024;
        if (di.smem_per_sm < di.max_smem_optin) di.smem_per_sm = di.max_smem_optin;
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_status_word) == cudaSuccess) g_status_ptr[dev] = static_cast<unsigned int*>(p);
        g_dev[dev] = di;
        g_dev_ready[dev].store(true, std::memory_order_release);
    }
    return g_dev[dev];
}

unsigned int* device_status_ptr() {
    const DeviceInfo& di = device_info();
    return g_status_ptr[di.device];
}

}  // namespace mlxq

using namespace mlxq;

extern "C" {

const char* mlxq_last_error(void) { return g_err.c_str(); }

int mlxq_quantize(const void* w_bf16, const mlxq_weight* dst, uint64_t stream) {
    WeightView v;
    int rc = check_weight(dst, v);
    if (rc) return rc;
    if (v.gs % 4 != 0)
        return fail(MLXQ_ERR_UNSUPPORTED, "quantize needs group_size %% 4 == 0 (got %lld)", static_cast<long long>(v.gs));
    if ((rc = check_buf(w_bf16, v.N * v.K, "w"))) return rc;
    const int64_t wbytes = v.N * v.K * 2, pbytes = v.N * v.K, tbytes = v.N * v.G * 2;
    if (overlap(w_bf16, wbytes, v.packed, pbytes) || overlap(w_bf16, wbytes, v.scales, tbytes) ||
        overlap(w_bf16, wbytes, v.biases, tbytes) || overlap(v.packed, pbytes, v.scales, tbytes) ||
        overlap(v.packed, pbytes, v.biases, tbytes) || overlap(v.scales, tbytes, v.biases, tbytes))
        return fail(MLXQ_ERR_INVALID_ARG, "quantize source and destination buffers overlap");
    if (v.N == 0 || v.K == 0) return ok();
    return launch_status(launch_quantize(w_bf16, v, as_stream(stream)), "quantize launch");
}

int mlxq_selftest_fail_alloc(uint32_t nth) {
    g_fail_alloc_in.store(static_cast<int>(nth > 1000000u ? 1000000u : nth));
    return ok();
}

int mlxq_selftest_wait_timeout(uint32_t limit_us, uint64_t stream) {
    if (limit_us < 1 || limit_us > 1000000u)
        return fail(MLXQ_ERR_INVALID_ARG, "limit_us must be in [1, 1000000], got %u", limit_us);
    return launch_status(launch_wait_timeout_selftest(1000ull * limit_us, as_stream(stream)),
                         "wait-timeout self-test launch");
}

int mlxq_load(const void* blob, size_t blob_len, const char* base, uint32_t group_size, mlxq_weight* out) {
    if (!out) return fail(MLXQ_ERR_INVALID_ARG, "null output handle");
    memset(out, 0, sizeof(*out));
    if (!blob || !base) return fail(MLXQ_ERR_INVALID_ARG, "null blob or base name");
    std::map<std::string, TensorInfo> ts;
    const uint8_t* data = nullptr;
    size_t data_len = 0;
    int rc = parse_safetensors(static_cast<const uint8_t*>(blob), blob_len, ts, data, data_len);
    if (rc != MLXQ_OK) return rc;
    const std::string b(base);
    const std::string names[3] = {b + ".weight", b + ".scales", b + ".biases"};
    for (const auto& n : names)
        if (!ts.count(n)) return fail(MLXQ_ERR_MISSING_TENSOR, "tensor '%s' is missing", n.c_str());
    const TensorInfo& tw = ts[names[0]];
    const TensorInfo& tsc = ts[names[1]];
    const TensorInfo& tb = ts[names[2]];
    if (tw.dtype != "U32") return fail(MLXQ_ERR_DTYPE, "'%s' has dtype %s, expected U32", names[0].c_str(), tw.dtype.c_str());
    if (tw.shape.size() != 2)
        return fail(MLXQ_ERR_SHAPE, "'%s' is %zu-D, expected 2-D", names[0].c_str(), tw.shape.size());
    const long long N = tw.shape[0], K = 4 * tw.shape[1];
    if (N > 0xFFFFFFFFLL || K > 0xFFFFFFFFLL) return fail(MLXQ_ERR_SHAPE, "'%s' is too large", names[0].c_str());
    if (group_size == 0 || K % group_size != 0)
        return fail(MLXQ_ERR_GROUP_SIZE, "group_size %u does not divide in_features %lld", group_size, K);
    const long long G = K / group_size;
    for (const TensorInfo* t : {&tsc, &tb}) {
        const std::string& nm = (t == &tsc) ? names[1] : names[2];
        if (t->dtype != "BF16") return fail(MLXQ_ERR_DTYPE, "'%s' has dtype %s, expected BF16", nm.c_str(), t->dtype.c_str());
        if (t->shape.size() != 2 || t->shape[0] != N || t->shape[1] != G)
            return fail(MLXQ_ERR_SHAPE, "'%s' must be [%lld, %lld]", nm.c_str(), N, G);
    }
    // allocate and upload (each buffer at least 256 bytes so an empty weight
    // still gets valid, non-null device pointers)
    const size_t bytes[3] = {static_cast<size_t>(N * K), static_cast<size_t>(N * G * 2), static_cast<size_t>(N * G * 2)};
    const TensorInfo* src[3] = {&tw, &tsc, &tb};
    void* ptr[3] = {nullptr, nullptr, nullptr};
    for (int i = 0; i < 3; ++i) {
        cudaError_t e = take_injected_alloc_failure() ? cudaErrorMemoryAllocation
                                                      : cudaMalloc(&ptr[i], bytes[i] < 256 ? 256 : bytes[i]);
        if (e == cudaSuccess && bytes[i]) e = cudaMemcpy(ptr[i], data + src[i]->begin, bytes[i], cudaMemcpyHostToDevice);
        if (e != cudaSuccess) {
            for (int j = 0; j <= i; ++j)
                if (ptr[j]) cudaFree(ptr[j]);
            return fail(MLXQ_ERR_CUDA, "uploading '%s': %s", names[i].c_str(), cudaGetErrorString(e));
        }
    }
    out->packed = ptr[0];
    out->scales = ptr[1];
    out->biases = ptr[2];
    out->out_features = static_cast<uint32_t>(N);
    out->in_features = static_cast<uint32_t>(K);
    out->group_size = group_size;
    out->flags = 0;
    return ok();
}

int mlxq_release(mlxq_weight* w) {
    if (!w) return fail(MLXQ_ERR_INVALID_ARG, "null weight handle");
    if (!w->packed && !w->scales && !w->biases)
        return fail(MLXQ_ERR_INVALID_ARG, "weight handle already released (release it once)");
    cudaError_t e = cudaSuccess, e2;
    void* ps[3] = {w->packed, w->scales, w->biases};
    for (void* p : ps)
        if (p && (e2 = cudaFree(p)) != cudaSuccess && e == cudaSuccess) e = e2;
    memset(w, 0, sizeof(*w));
    return launch_status(e, "cudaFree");
}

int mlxq_dequant(const mlxq_weight* w, void* out, uint64_t stream) {
    WeightView v;
    int rc = check_weight(w, v);
    if (rc) return rc;
    if ((rc = check_buf(out, v.N * v.K, "out"))) return rc;
    if ((rc = check_out_vs_weight(out, v.N * v.K * 2, v))) return rc;
    return launch_status(launch_dequant(v, out, as_stream(stream)), "mlx_int8_dequant launch");
}

int mlxq_dequant_as(const mlxq_weight* w, void* out, int dtype, uint64_t stream) {
    WeightView v;
    int rc = check_weight(w, v);
    if (rc) return rc;
    if (dtype < MLXQ_DTYPE_BF16 || dtype > MLXQ_DTYPE_F32) return fail(MLXQ_ERR_INVALID_ARG, "unknown dtype %d", dtype);
    const int64_t esize = dtype == MLXQ_DTYPE_F32 ? 4 : 2;
    if (v.N * v.K != 0) {
        if (!out) return fail(MLXQ_ERR_INVALID_ARG, "out is null");
        if (!aligned(out, static_cast<size_t>(esize))) return fail(MLXQ_ERR_INVALID_ARG, "out is not %lld-byte aligned",
                                                                    static_cast<long long>(esize));
    }
    if ((rc = check_out_vs_weight(out, v.N * v.K * esize, v))) return rc;
    return launch_status(launch_dequant_as(v, out, dtype, as_stream(stream)), "dequant launch");
}

static int gemv_common(const mlxq_weight* w, int mode, const void* x, const void* gate, const void* up,
                       const void* resid, void* y, uint64_t stream) {
    WeightView v;
    int rc = check_weight(w, v);
    if (rc) return rc;
    if (mode == GEMV_PLAIN) {
        if ((rc = check_buf(x, v.K, "x"))) return rc;
    } else {
        if ((rc = check_buf(gate, v.K, "gate"))) return rc;
        if ((rc = check_buf(up, v.K, "up"))) return rc;
    }
    if (mode == GEMV_SILU_RESID && (rc = check_buf(resid, v.N, "x_resid"))) return rc;
    if ((rc = check_buf(y, v.N, "y"))) return rc;
    const int64_t yb = v.N * 2, kb = v.K * 2;
    if (overlap(y, yb, x, kb) || overlap(y, yb, gate, kb) || overlap(y, yb, up, kb))
        return fail(MLXQ_ERR_INVALID_ARG, "y overlaps an input vector");
    if (mode == GEMV_SILU_RESID && resid != y && overlap(y, yb, resid, yb))
        return fail(MLXQ_ERR_INVALID_ARG, "y overlaps x_resid without being equal to it");
    if ((rc = check_out_vs_weight(y, yb, v))) return rc;
    if (v.N == 0) return ok();
    return launch_status(launch_gemv(v, mode, x, gate, up, resid, y, as_stream(stream)), "gemv launch");
}

int mlxq_gemv(const mlxq_weight* w, const void* x, void* y, uint64_t stream) {
    return gemv_common(w, GEMV_PLAIN, x, nullptr, nullptr, nullptr, y, stream);
}

int mlxq_gemv_silu_gate(const mlxq_weight* w, const void* gate, const void* up, void* y, uint64_t stream) {
    return gemv_common(w, GEMV_SILU, nullptr, gate, up, nullptr, y, stream);
}

int mlxq_gemv_silu_gate_resid(const mlxq_weight* w, const void* gate, const void* up, const void* x_resid,
                              void* y, uint64_t stream) {
    return gemv_common(w, GEMV_SILU_RESID, nullptr, gate, up, x_resid, y, stream);
}

// Kernel choice by m: the weight-streaming kernels read every weight byte
// once and are HBM-bound while the per-byte work fits the SM; beyond
// kStreamMmaMaxM rows the tcgen05 kernel takes over.
namespace {

int gemm_impl(const mlxq_weight* w, const void* x, void* y, uint32_t m, int kernel, uint64_t stream,
              TcScratch scratch) {
    WeightView v;
    int rc = check_weight(w, v);
    if (rc) return rc;
    if (kernel < MLXQ_GEMM_AUTO || kernel > MLXQ_GEMM_SMALLM_TC)
        return fail(MLXQ_ERR_INVALID_ARG, "unknown gemm kernel id %d", kernel);
    if (m == 0) return ok();
    const int64_t M = m;
    if ((v.K > v.N ? v.K : v.N) > (int64_t{1} << 50) / M)
        return fail(MLXQ_ERR_SHAPE, "m x in_features or m x out_features is beyond any device");
    if ((rc = check_buf(x, M * v.K, "X"))) return rc;
    if ((rc = check_buf(y, M * v.N, "Y"))) return rc;
    if (overlap(y, M * v.N * 2, x, M * v.K * 2)) return fail(MLXQ_ERR_INVALID_ARG, "Y overlaps X");
    if ((rc = check_out_vs_weight(y, M * v.N * 2, v))) return rc;
    if (v.N == 0) return ok();
    cudaStream_t s = as_stream(stream);
    const bool x16 = (reinterpret_cast<uintptr_t>(x) & 15u) == 0;
    int k = kernel;
    if (k == MLXQ_GEMM_AUTO) {
        if (M == 1) k = MLXQ_GEMM_ROWS;
        else if (smallm_tc_preferred(v, M, x)) k = MLXQ_GEMM_SMALLM_TC;
        else if (M <= kStreamMmaMaxM && smallm_preferred(v, M, x)) k = MLXQ_GEMM_SMALLM_GROUPS;
        else if (M <= kStreamMmaMaxM && stream_mma_supported(v, GEMV_PLAIN, M, x, nullptr, nullptr))
            k = MLXQ_GEMM_SMALLM;
        else if (smallm_supported(v, M, x)) k = MLXQ_GEMM_SMALLM_GROUPS;
        else if (gemm_tc_supported(v, M, x, y)) k = MLXQ_GEMM_TCGEN05;
        else if ((M <= kSmallMMax && x16 && gemm_smallm_supported(v, M)) || anygs_gemm_supported(v, M))
            k = MLXQ_GEMM_SMALLM_FFMA;
        else k = MLXQ_GEMM_ROWS;
    }
    switch (k) {
        case MLXQ_GEMM_ROWS: {
            const uint16_t* X = static_cast<const uint16_t*>(x);
            uint16_t* Y = static_cast<uint16_t*>(y);
            for (int64_t i = 0; i < M; ++i) {
                cudaError_t e = launch_gemv(v, GEMV_PLAIN, X + i * v.K, nullptr, nullptr, nullptr, Y + i * v.N, s);
                if (e != cudaSuccess) return launch_status(e, "gemm (row passes) launch");
            }
            return ok();
        }
        case MLXQ_GEMM_SMALLM_TC:
            if (!smallm_tc_supported(v, M, x))
                return fail(MLXQ_ERR_UNSUPPORTED, "small-m tcgen05 kernel cannot take m=%lld, K=%lld, group_size=%lld",
                            static_cast<long long>(M), static_cast<long long>(v.K), static_cast<long long>(v.gs));
            return launch_status(launch_smallm_tc(v, x, y, M, s), "small-m tcgen05 gemm launch");
        case MLXQ_GEMM_SMALLM_GROUPS:
            if (!smallm_supported(v, M, x))
                return fail(MLXQ_ERR_UNSUPPORTED, "small-m tile-group kernel cannot take m=%lld, K=%lld, group_size=%lld",
                            static_cast<long long>(M), static_cast<long long>(v.K), static_cast<long long>(v.gs));
            return launch_status(launch_smallm(v, x, y, M, s), "small-m tile-group gemm launch");
        case MLXQ_GEMM_SMALLM:
            if (M > kStreamMmaMaxM || !stream_mma_supported(v, GEMV_PLAIN, M, x, nullptr, nullptr))
                return fail(MLXQ_ERR_UNSUPPORTED, "small-m tensor-pipe kernel cannot take m=%lld, K=%lld, group_size=%lld",
                            static_cast<long long>(M), static_cast<long long>(v.K), static_cast<long long>(v.gs));
            return launch_status(launch_stream_mma(v, GEMV_PLAIN, M, x, nullptr, nullptr, nullptr, y, s),
                                 "small-m gemm launch");
        case MLXQ_GEMM_SMALLM_FFMA:
            if (M <= kSmallMMax && x16 && gemm_smallm_supported(v, M))
                return launch_status(launch_gemm_smallm(v, x, y, M, s), "small-m fp32 gemm launch");
            if (anygs_gemm_supported(v, M))
                return launch_status(launch_anygs_gemm(v, x, y, M, s), "small-m fp32 gemm (any group size) launch");
            {
                return fail(MLXQ_ERR_UNSUPPORTED, "small-m fp32 kernel cannot take m=%lld, K=%lld, group_size=%lld",
                            static_cast<long long>(M), static_cast<long long>(v.K), static_cast<long long>(v.gs));
            }
        default:
            if (!gemm_tc_supported(v, M, x, y))
                return fail(MLXQ_ERR_UNSUPPORTED, "tensor-core kernel cannot take m=%lld, N=%lld, K=%lld, group_size=%lld",
                            static_cast<long long>(M), static_cast<long long>(v.N), static_cast<long long>(v.K),
                            static_cast<long long>(v.gs));
            if (scratch == TC_SCRATCH_STATIC && gemm_tc_scratch_bytes(v, M) > kStaticScratchBytes)
                return fail(MLXQ_ERR_UNSUPPORTED, "K split of m=%lld, N=%lld needs %zu bytes of scratch; the static buffer holds %zu",
                            static_cast<long long>(M), static_cast<long long>(v.N), gemm_tc_scratch_bytes(v, M),
                            kStaticScratchBytes);
            return launch_status(launch_gemm_tc(v, x, y, M, s, scratch), "tcgen05 gemm launch");
    }
}

}  // namespace

int mlxq_gemm_with(const mlxq_weight* w, const void* x, void* y, uint32_t m, int kernel, uint64_t stream) {
    return gemm_impl(w, x, y, m, kernel, stream, TC_SCRATCH_POOL);
}

int mlxq_gemm(const mlxq_weight* w, const void* x, void* y, uint32_t m, uint64_t stream) {
    return gemm_impl(w, x, y, m, MLXQ_GEMM_AUTO, stream, TC_SCRATCH_POOL);
}

int mlxq_gemm_noalloc(const mlxq_weight* w, const void* x, void* y, uint32_t m, uint64_t stream) {
    return gemm_impl(w, x, y, m, MLXQ_GEMM_AUTO, stream, TC_SCRATCH_STATIC);
}

int mlxq_device_status(void) {
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return launch_status(e, "cudaDeviceSynchronize");
    unsigned int v = 0, zero = 0;
    e = cudaMemcpyFromSymbol(&v, g_status_word, sizeof(v));
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_status_word, &zero, sizeof(zero));
    if (e != cudaSuccess) return launch_status(e, "reading the device status word");
    if (v) {
        // a split gemm may have stopped between raising and clearing its tile
        // counters: zero the static scratch's counters so mlxq_gemm_noalloc
        // starts clean again
        e = reset_static_scratch_counters();
        if (e != cudaSuccess) return launch_status(e, "resetting the static scratch counters");
        return fail(MLXQ_ERR_DEVICE_TIMEOUT, "a kernel gave up a bounded pipeline wait (status 0x%x)", v);
    }
    return ok();
}

}  // extern "C"

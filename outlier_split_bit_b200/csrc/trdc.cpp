// trdc.cpp -- the TRDC container: writer and streaming loader (host code).
//
// Method: "SPECTRA: Sparse-Precision Exact Channel Tensor Reconstruction
// Architecture" (Dev.to abstract), abstract paragraph: every weight, scale
// and offset is serialised into one self-contained binary container that is
// streamed straight into GPU memory, so that initialisation has a bounded
// memory spike.  The byte format (spectra.h) is the library's own.
//
// Streaming: a buffer moves through the caller's staging buffer in chunks of
// half its size.  Loading, the file read of chunk j (pread into one half)
// overlaps the host-to-device copy of chunk j - 1 (from the other half, on
// the caller's stream); a half is refilled only after the event recorded
// behind its previous copy has completed.  Writing runs the mirror image.
// Host memory in use is the staging buffer and the reader handle (the layer
// records), whatever the size of the model.  With SPECTRA_MEM_HOST the
// buffers are host memory and no CUDA call is made.
#include <cuda_runtime.h>
#include <fcntl.h>
#include <sys/stat.h>
#include <unistd.h>

#include <cerrno>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <thread>

#include "internal.cuh"
#include "spectra.h"

struct spectra_trdc {
    int fd;
    int32_t count;
    uint64_t file_bytes;
    spectra_trdc_layer *rec;
};

namespace spectra {
namespace {

constexpr uint32_t kVersion = 1;
constexpr size_t kHeaderBytes = 64;
constexpr size_t kRecordBytes = 256;
constexpr uint64_t kAlign = 4096;
constexpr size_t kMinStaging = 8192;
constexpr int kBuffers = 6;  // codes, scales, zeros, outlier_idx, outlier_w, bulk_idx

// ---------------------------------------------------------------- CRC-32

// Reflected CRC-32 with the IEEE polynomial, eight bytes per step (the
// "slicing" tables: tab[t][b] is the CRC contribution of byte b followed by
// t zero bytes).  Buffers of 4 MB and more are split over up to eight
// threads and the slices' CRCs combined (crc_concat).
uint32_t g_tab[8][256];
std::once_flag g_tab_once;

void build_tables() {
    for (uint32_t i = 0; i < 256; ++i) {
        uint32_t c = i;
        for (int b = 0; b < 8; ++b) c = (c & 1u) ? (0xEDB88320u ^ (c >> 1)) : (c >> 1);
        g_tab[0][i] = c;
    }
    for (uint32_t i = 0; i < 256; ++i)
        for (int t = 1; t < 8; ++t) g_tab[t][i] = (g_tab[t - 1][i] >> 8) ^ g_tab[0][g_tab[t - 1][i] & 0xFFu];
}

// Advances the register state (not inverted) over n bytes.
uint32_t crc_step(uint32_t s, const uint8_t *p, size_t n) {
    while (n >= 8) {
        uint32_t lo, hi;
        std::memcpy(&lo, p, 4);
        std::memcpy(&hi, p + 4, 4);
        lo ^= s;
        s = g_tab[7][lo & 0xFFu] ^ g_tab[6][(lo >> 8) & 0xFFu] ^ g_tab[5][(lo >> 16) & 0xFFu] ^
            g_tab[4][lo >> 24] ^ g_tab[3][hi & 0xFFu] ^ g_tab[2][(hi >> 8) & 0xFFu] ^
            g_tab[1][(hi >> 16) & 0xFFu] ^ g_tab[0][hi >> 24];
        p += 8;
        n -= 8;
    }
    while (n--) s = (s >> 8) ^ g_tab[0][(s ^ *p++) & 0xFFu];
    return s;
}

uint32_t crc_serial(uint32_t prev, const void *data, size_t n) {
    std::call_once(g_tab_once, build_tables);
    return ~crc_step(~prev, static_cast<const uint8_t *>(data), n);
}

// Multiplication modulo the CRC polynomial in the reflected representation
// (bit 31 is the coefficient of x^0, bit 0 that of x^31).
uint32_t mulmod(uint32_t a, uint32_t b) {
    uint32_t p = 0;
    for (uint32_t m = 1u << 31; m; m >>= 1) {
        if (a & m) p ^= b;
        b = (b & 1u) ? (b >> 1) ^ 0xEDB88320u : b >> 1;  // b *= x
    }
    return p;
}

// x^(8n) modulo the polynomial: the operator that runs a CRC register
// through n zero bytes.
uint32_t x8n(uint64_t n) {
    uint32_t r = 1u << 31;          // 1
    uint32_t sq = 1u << 23;         // x^8
    for (; n; n >>= 1) {
        if (n & 1u) r = mulmod(r, sq);
        sq = mulmod(sq, sq);
    }
    return r;
}

// CRC of A followed by B from the CRCs of the two parts: the register of A,
// run through |B| zero bytes, XOR the CRC of B (the initial and final
// inversions cancel out of the combination).
uint32_t crc_concat(uint32_t crc_a, uint32_t crc_b, uint64_t len_b) {
    return mulmod(x8n(len_b), crc_a) ^ crc_b;
}

// Large buffers are checksummed in slices on several threads and combined.
constexpr size_t kParallelCrcBytes = 4u << 20;

uint32_t crc(uint32_t prev, const void *data, size_t n) {
    const unsigned hw = std::thread::hardware_concurrency();
    if (n < kParallelCrcBytes || hw < 2) return crc_serial(prev, data, n);
    std::call_once(g_tab_once, build_tables);
    size_t parts = n / (1u << 20);
    if (parts > 8) parts = 8;
    if (parts > hw) parts = hw;
    const size_t slice = (n / parts + 63) & ~(size_t)63;
    uint32_t part_crc[8] = {0};
    size_t part_len[8] = {0};
    std::thread pool[8];
    const uint8_t *p = static_cast<const uint8_t *>(data);
    size_t used = 0;
    for (size_t i = 0; i < parts; ++i) {
        const size_t len = (i + 1 == parts) ? n - used : (slice < n - used ? slice : n - used);
        part_len[i] = len;
        const uint8_t *q = p + used;
        uint32_t *out = &part_crc[i];
        pool[i] = std::thread([q, len, out] { *out = crc_serial(0, q, len); });
        used += len;
    }
    uint32_t c = prev;
    for (size_t i = 0; i < parts; ++i) {
        pool[i].join();
        c = crc_concat(c, part_crc[i], part_len[i]);
    }
    return c;
}

// ---------------------------------------------------------------- layout

template <typename T>
void put(uint8_t *dst, size_t off, T v) {
    std::memcpy(dst + off, &v, sizeof v);
}
template <typename T>
T get(const uint8_t *src, size_t off) {
    T v;
    std::memcpy(&v, src + off, sizeof v);
    return v;
}

uint64_t align_up(uint64_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Expected byte sizes of a layer's six buffers (0 for absent ones), or a
// failed status for an impossible shape.
spectra_status buffer_sizes(int32_t n, int32_t k, int32_t n_o, bool compact, uint64_t sizes[kBuffers],
                            int32_t *k_bulk) {
    spectra_sizes sz;
    const spectra_status st = compact ? spectra_packed_sizes_compact(n, k, n_o, &sz)
                                      : spectra_packed_sizes(n, k, n_o, &sz);
    if (st != SPECTRA_OK) return st;
    sizes[0] = sz.codes_bytes;
    sizes[1] = sz.scales_bytes;
    sizes[2] = sz.zeros_bytes;
    sizes[3] = n_o > 0 ? sz.outlier_idx_bytes : 0;
    sizes[4] = n_o > 0 ? sz.outlier_w_bytes : 0;
    sizes[5] = compact ? sz.bulk_idx_bytes : 0;
    *k_bulk = compact ? sz.k_bulk : 0;
    return SPECTRA_OK;
}

void encode_record(const spectra_trdc_layer &r, uint8_t *dst) {
    std::memset(dst, 0, kRecordBytes);
    std::memcpy(dst, r.name, 96);
    put<int32_t>(dst, 96, r.n);
    put<int32_t>(dst, 100, r.k);
    put<int32_t>(dst, 104, r.n_outliers);
    put<int32_t>(dst, 108, r.k_bulk);
    put<double>(dst, 112, r.tau);
    put<uint32_t>(dst, 120, r.flags);
    for (int b = 0; b < kBuffers; ++b) {
        put<uint64_t>(dst, 128 + 16 * b, r.offset[b]);
        put<uint64_t>(dst, 136 + 16 * b, r.bytes[b]);
        put<uint32_t>(dst, 224 + 4 * b, r.crc32[b]);
    }
}

void decode_record(const uint8_t *src, spectra_trdc_layer *r) {
    std::memset(r, 0, sizeof *r);
    std::memcpy(r->name, src, 96);
    r->name[95] = '\0';
    r->n = get<int32_t>(src, 96);
    r->k = get<int32_t>(src, 100);
    r->n_outliers = get<int32_t>(src, 104);
    r->k_bulk = get<int32_t>(src, 108);
    r->tau = get<double>(src, 112);
    r->flags = get<uint32_t>(src, 120);
    for (int b = 0; b < kBuffers; ++b) {
        r->offset[b] = get<uint64_t>(src, 128 + 16 * b);
        r->bytes[b] = get<uint64_t>(src, 136 + 16 * b);
        r->crc32[b] = get<uint32_t>(src, 224 + 4 * b);
    }
}

bool pwrite_all(int fd, const void *p, size_t n, uint64_t off) {
    const uint8_t *q = static_cast<const uint8_t *>(p);
    while (n > 0) {
        const ssize_t w = ::pwrite(fd, q, n, (off_t)off);
        if (w < 0 && errno == EINTR) continue;
        if (w <= 0) return false;
        q += w;
        n -= (size_t)w;
        off += (uint64_t)w;
    }
    return true;
}

bool pread_all(int fd, void *p, size_t n, uint64_t off) {
    uint8_t *q = static_cast<uint8_t *>(p);
    while (n > 0) {
        const ssize_t r = ::pread(fd, q, n, (off_t)off);
        if (r < 0 && errno == EINTR) continue;
        if (r <= 0) return false;
        q += r;
        n -= (size_t)r;
        off += (uint64_t)r;
    }
    return true;
}

// Two events behind the two staging halves, created for one call (only for
// device memory: host-memory calls make no CUDA call).
struct Halves {
    cudaEvent_t ev[2] = {nullptr, nullptr};
    bool ok = true;
    explicit Halves(bool create) {
        if (create)
            ok = cudaEventCreateWithFlags(&ev[0], cudaEventDisableTiming) == cudaSuccess &&
                 cudaEventCreateWithFlags(&ev[1], cudaEventDisableTiming) == cudaSuccess;
    }
    Halves(const Halves &) = delete;
    Halves &operator=(const Halves &) = delete;
    ~Halves() {
        for (cudaEvent_t e : ev)
            if (e) cudaEventDestroy(e);
    }
};

// How chunks move between a staging half and the caller's buffer: on the
// caller's stream with an event behind each half (device memory), or by
// memcpy (host memory, which makes the same chunk loop testable without a
// GPU).
struct DeviceCopier {
    Halves &h;
    cudaStream_t s;
    spectra_status wait(int k) {
        return cudaEventSynchronize(h.ev[k]) == cudaSuccess ? SPECTRA_OK : SPECTRA_ERR_CUDA;
    }
    spectra_status copy(void *dst, const void *src, size_t n, bool to_device, int k) {
        if (cudaMemcpyAsync(dst, src, n, to_device ? cudaMemcpyHostToDevice : cudaMemcpyDeviceToHost,
                            s) != cudaSuccess ||
            cudaEventRecord(h.ev[k], s) != cudaSuccess)
            return SPECTRA_ERR_CUDA;
        return SPECTRA_OK;
    }
    // after a failure: let the copies still using the staging buffer finish
    void drain() {
        cudaEventSynchronize(h.ev[0]);
        cudaEventSynchronize(h.ev[1]);
    }
};

struct HostCopier {
    spectra_status wait(int) { return SPECTRA_OK; }
    spectra_status copy(void *dst, const void *src, size_t n, bool, int) {
        std::memcpy(dst, src, n);
        return SPECTRA_OK;
    }
    void drain() {}
};

// Checksum of one staged chunk, computed on a thread of its own.
struct CrcJob {
    std::thread t;
    uint32_t value = 0;
    size_t len = 0;
    bool active = false;
    void start(const uint8_t *p, size_t n) {
        len = n;
        active = true;
        t = std::thread([this, p, n] { value = crc(0, p, n); });
    }
    // folds this chunk into the running CRC (chunks must be folded in order)
    void finish(uint32_t *running) {
        if (!active) return;
        t.join();
        *running = crc_concat(*running, value, len);
        active = false;
    }
    ~CrcJob() {
        if (t.joinable()) t.join();
    }
};

// One buffer from the file into the caller's memory through the staging
// halves.  Chunk j: wait until half j % 2 is free (its copy and its checksum
// done), read the chunk into it, start its copy, and checksum it on a
// thread while chunk j + 1 is read into the other half.  Checksums are
// folded into the running CRC in chunk order.
template <typename Copier>
spectra_status load_buffer(int fd, uint64_t off, uint64_t bytes, uint8_t *dst, uint8_t *staging,
                           size_t half, bool verify, uint32_t *crc_out, Copier &cp) {
    uint32_t c = 0;
    bool pending[2] = {false, false};
    CrcJob job[2];
    spectra_status st = SPECTRA_OK;
    for (uint64_t done = 0, j = 0; done < bytes && st == SPECTRA_OK; done += half, ++j) {
        const int k = (int)(j & 1);
        const size_t len = (size_t)((bytes - done) < half ? (bytes - done) : half);
        if (pending[k] && (st = cp.wait(k)) != SPECTRA_OK) break;
        job[k].finish(&c);  // chunk j - 2 (chunk j - 1, if any, is still running)
        uint8_t *buf = staging + (size_t)k * half;
        if (!pread_all(fd, buf, len, off + done)) {
            st = SPECTRA_ERR_IO;
            break;
        }
        st = cp.copy(dst + done, buf, len, true, k);
        pending[k] = true;
        if (verify && st == SPECTRA_OK) job[k].start(buf, len);
    }
    // fold the remaining chunks in order: the earlier one is in the half of
    // the second-to-last chunk
    const uint64_t nchunks = bytes == 0 ? 0 : (bytes + half - 1) / half;
    if (nchunks >= 2) job[(nchunks - 2) & 1].finish(&c);
    if (nchunks >= 1) job[(nchunks - 1) & 1].finish(&c);
    for (int k = 0; k < 2 && st == SPECTRA_OK; ++k)
        if (pending[k]) st = cp.wait(k);
    if (st != SPECTRA_OK) {
        job[0].finish(&c);
        job[1].finish(&c);
        cp.drain();
        return st;
    }
    *crc_out = c;
    return SPECTRA_OK;
}

// One buffer from the caller's memory into the file through the staging
// halves: the copy of chunk j overlaps the file write of chunk j - 1.
template <typename Copier>
spectra_status write_buffer(int fd, uint64_t off, uint64_t bytes, const uint8_t *src,
                            uint8_t *staging, size_t half, uint32_t *crc_out, Copier &cp) {
    uint32_t c = 0;
    uint64_t prev_done = 0;
    size_t prev_len = 0;
    int prev_k = 0;
    spectra_status st = SPECTRA_OK;
    for (uint64_t done = 0, j = 0; done < bytes; done += half, ++j) {
        const int k = (int)(j & 1);
        const size_t len = (size_t)((bytes - done) < half ? (bytes - done) : half);
        if ((st = cp.copy(staging + (size_t)k * half, src + done, len, false, k)) != SPECTRA_OK) break;
        if (j > 0) {
            uint8_t *pb = staging + (size_t)prev_k * half;
            if ((st = cp.wait(prev_k)) != SPECTRA_OK) break;
            c = crc(c, pb, prev_len);
            if (!pwrite_all(fd, pb, prev_len, off + prev_done)) {
                st = SPECTRA_ERR_IO;
                break;
            }
        }
        prev_done = done;
        prev_len = len;
        prev_k = k;
    }
    if (st == SPECTRA_OK && bytes > 0) {
        uint8_t *pb = staging + (size_t)prev_k * half;
        if ((st = cp.wait(prev_k)) == SPECTRA_OK) {
            c = crc(c, pb, prev_len);
            if (!pwrite_all(fd, pb, prev_len, off + prev_done)) st = SPECTRA_ERR_IO;
        }
    }
    if (st != SPECTRA_OK) {
        cp.drain();
        return st;
    }
    *crc_out = c;
    return SPECTRA_OK;
}

const void *layer_buffer(const spectra_layer &l, int b) {
    switch (b) {
        case 0: return l.codes;
        case 1: return l.scales;
        case 2: return l.zeros;
        case 3: return l.outlier_idx;
        case 4: return l.outlier_w;
        default: return l.bulk_idx;
    }
}

}  // namespace
}  // namespace spectra

using namespace spectra;

extern "C" {

uint32_t spectra_crc32(uint32_t prev, const void *data, size_t bytes) {
    if (!data || bytes == 0) return prev;
    return crc(prev, data, bytes);
}

spectra_status spectra_trdc_write(const char *path, int32_t count, const char *const *names,
                                  const spectra_layer *layers, const double *taus,
                                  spectra_memory mem, void *staging, size_t staging_bytes,
                                  void *stream) {
    if (!path || !names || !layers || count < 1 || count > (1 << 20)) return SPECTRA_ERR_INVALID_ARG;
    if (mem != SPECTRA_MEM_DEVICE && mem != SPECTRA_MEM_HOST) return SPECTRA_ERR_INVALID_ARG;
    if (mem == SPECTRA_MEM_DEVICE && !staging) return SPECTRA_ERR_INVALID_ARG;
    if (staging && staging_bytes < kMinStaging) return SPECTRA_ERR_BUFFER_TOO_SMALL;
    // records and file placement, before anything is written
    spectra_trdc_layer *rec = static_cast<spectra_trdc_layer *>(std::calloc((size_t)count, sizeof *rec));
    if (!rec) return SPECTRA_ERR_INTERNAL;
    uint64_t pos = kHeaderBytes + kRecordBytes * (uint64_t)count;
    for (int32_t i = 0; i < count; ++i) {
        const spectra_layer &l = layers[i];
        const bool compact = l.bulk_idx != nullptr;
        spectra_trdc_layer &r = rec[i];
        if (!names[i] || std::strlen(names[i]) >= sizeof r.name) {
            std::free(rec);
            return SPECTRA_ERR_INVALID_ARG;
        }
        std::strncpy(r.name, names[i], sizeof r.name - 1);
        r.n = l.n;
        r.k = l.k;
        r.n_outliers = l.n_outliers;
        r.tau = taus ? taus[i] : 0.0;
        r.flags = compact ? 1u : 0u;
        uint64_t sizes[kBuffers];
        const spectra_status st = buffer_sizes(l.n, l.k, l.n_outliers, compact, sizes, &r.k_bulk);
        if (st != SPECTRA_OK || (compact && l.k_bulk != r.k_bulk)) {
            std::free(rec);
            return st != SPECTRA_OK ? st : SPECTRA_ERR_INVALID_ARG;
        }
        for (int b = 0; b < kBuffers; ++b) {
            r.bytes[b] = sizes[b];
            if (sizes[b] == 0) continue;
            if (!layer_buffer(l, b)) {
                std::free(rec);
                return SPECTRA_ERR_INVALID_ARG;
            }
            r.offset[b] = align_up(pos);
            pos = r.offset[b] + sizes[b];
        }
    }
    const uint64_t file_bytes = pos;
    const int fd = ::open(path, O_WRONLY | O_CREAT | O_TRUNC, 0644);
    if (fd < 0) {
        std::free(rec);
        return SPECTRA_ERR_IO;
    }
    spectra_status st = SPECTRA_OK;
    {
        Halves h(mem == SPECTRA_MEM_DEVICE);
        if (!h.ok) st = SPECTRA_ERR_CUDA;
        const size_t half = (staging_bytes / 2) & ~(size_t)15;
        for (int32_t i = 0; i < count && st == SPECTRA_OK; ++i)
            for (int b = 0; b < kBuffers && st == SPECTRA_OK; ++b) {
                spectra_trdc_layer &r = rec[i];
                if (r.bytes[b] == 0) continue;
                const uint8_t *src = static_cast<const uint8_t *>(layer_buffer(layers[i], b));
                uint8_t *stg = static_cast<uint8_t *>(staging);
                if (mem == SPECTRA_MEM_DEVICE) {
                    DeviceCopier cp{h, (cudaStream_t)stream};
                    st = write_buffer(fd, r.offset[b], r.bytes[b], src, stg, half, &r.crc32[b], cp);
                } else if (staging) {
                    HostCopier cp;
                    st = write_buffer(fd, r.offset[b], r.bytes[b], src, stg, half, &r.crc32[b], cp);
                } else {
                    r.crc32[b] = crc(0, src, (size_t)r.bytes[b]);
                    if (!pwrite_all(fd, src, (size_t)r.bytes[b], r.offset[b])) st = SPECTRA_ERR_IO;
                }
            }
    }
    if (st == SPECTRA_OK) {
        const size_t hb = kHeaderBytes + kRecordBytes * (size_t)count;
        uint8_t *head = static_cast<uint8_t *>(std::calloc(hb, 1));
        if (!head) {
            st = SPECTRA_ERR_INTERNAL;
        } else {
            for (int32_t i = 0; i < count; ++i) encode_record(rec[i], head + kHeaderBytes + kRecordBytes * i);
            std::memcpy(head, "TRDC", 4);
            put<uint32_t>(head, 4, kVersion);
            put<uint32_t>(head, 8, (uint32_t)count);
            put<uint32_t>(head, 12, (uint32_t)hb);
            put<uint64_t>(head, 16, file_bytes);
            put<uint32_t>(head, 24, crc(0, head + kHeaderBytes, kRecordBytes * (size_t)count));
            if (!pwrite_all(fd, head, hb, 0)) st = SPECTRA_ERR_IO;
            std::free(head);
        }
    }
    if (::close(fd) != 0 && st == SPECTRA_OK) st = SPECTRA_ERR_IO;
    std::free(rec);
    return st;
}

spectra_status spectra_trdc_open(const char *path, spectra_trdc **out) {
    if (!path || !out) return SPECTRA_ERR_INVALID_ARG;
    const int fd = ::open(path, O_RDONLY);
    if (fd < 0) return SPECTRA_ERR_IO;
    struct stat stt;
    uint8_t head[kHeaderBytes];
    if (::fstat(fd, &stt) != 0) {
        ::close(fd);
        return SPECTRA_ERR_IO;
    }
    const uint64_t size = (uint64_t)stt.st_size;
    if (size < kHeaderBytes || !pread_all(fd, head, kHeaderBytes, 0)) {
        ::close(fd);
        return SPECTRA_ERR_FORMAT;
    }
    const uint32_t count = get<uint32_t>(head, 8);
    const uint64_t hb = kHeaderBytes + kRecordBytes * (uint64_t)count;
    if (std::memcmp(head, "TRDC", 4) != 0 || get<uint32_t>(head, 4) != kVersion || count < 1 ||
        count > (1u << 20) || get<uint32_t>(head, 12) != hb || get<uint64_t>(head, 16) != size ||
        hb > size) {
        ::close(fd);
        return SPECTRA_ERR_FORMAT;
    }
    uint8_t *raw = static_cast<uint8_t *>(std::malloc((size_t)(hb - kHeaderBytes)));
    spectra_trdc_layer *rec = static_cast<spectra_trdc_layer *>(std::calloc(count, sizeof *rec));
    spectra_status st = (raw && rec) ? SPECTRA_OK : SPECTRA_ERR_INTERNAL;
    if (st == SPECTRA_OK && !pread_all(fd, raw, (size_t)(hb - kHeaderBytes), kHeaderBytes)) st = SPECTRA_ERR_FORMAT;
    if (st == SPECTRA_OK && crc(0, raw, (size_t)(hb - kHeaderBytes)) != get<uint32_t>(head, 24))
        st = SPECTRA_ERR_FORMAT;
    uint64_t end = hb;
    for (uint32_t i = 0; i < count && st == SPECTRA_OK; ++i) {
        spectra_trdc_layer &r = rec[i];
        decode_record(raw + kRecordBytes * i, &r);
        if (r.flags > 1u || r.n_outliers < 0) {
            st = SPECTRA_ERR_FORMAT;
            break;
        }
        const bool compact = (r.flags & 1u) != 0;
        uint64_t sizes[kBuffers];
        int32_t kb = 0;
        if (buffer_sizes(r.n, r.k, r.n_outliers, compact, sizes, &kb) != SPECTRA_OK || kb != r.k_bulk) {
            st = SPECTRA_ERR_FORMAT;
            break;
        }
        for (int b = 0; b < kBuffers && st == SPECTRA_OK; ++b) {
            if (r.bytes[b] != sizes[b]) st = SPECTRA_ERR_FORMAT;
            else if (sizes[b] == 0 && (r.offset[b] != 0 || r.crc32[b] != 0)) st = SPECTRA_ERR_FORMAT;
            else if (sizes[b] > 0) {
                // buffers in file order, aligned, inside the file
                if (r.offset[b] % kAlign || r.offset[b] < end || r.offset[b] + r.bytes[b] > size)
                    st = SPECTRA_ERR_FORMAT;
                else
                    end = r.offset[b] + r.bytes[b];
            }
        }
    }
    std::free(raw);
    if (st != SPECTRA_OK) {
        std::free(rec);
        ::close(fd);
        return st;
    }
    spectra_trdc *t = static_cast<spectra_trdc *>(std::malloc(sizeof *t));
    if (!t) {
        std::free(rec);
        ::close(fd);
        return SPECTRA_ERR_INTERNAL;
    }
    t->fd = fd;
    t->count = (int32_t)count;
    t->file_bytes = size;
    t->rec = rec;
    *out = t;
    return SPECTRA_OK;
}

int32_t spectra_trdc_count(const spectra_trdc *t) { return t ? t->count : 0; }

spectra_status spectra_trdc_info(const spectra_trdc *t, int32_t i, spectra_trdc_layer *out) {
    if (!t || !out || i < 0 || i >= t->count) return SPECTRA_ERR_INVALID_ARG;
    *out = t->rec[i];
    return SPECTRA_OK;
}

spectra_status spectra_trdc_load(const spectra_trdc *t, int32_t i, uint8_t *codes, uint16_t *scales,
                                 uint32_t *zeros, int32_t *outlier_idx, uint16_t *outlier_w,
                                 int32_t *bulk_idx, spectra_memory mem, void *staging,
                                 size_t staging_bytes, int32_t verify, spectra_layer *layer_out,
                                 void *stream) {
    if (!t || i < 0 || i >= t->count) return SPECTRA_ERR_INVALID_ARG;
    if (mem != SPECTRA_MEM_DEVICE && mem != SPECTRA_MEM_HOST) return SPECTRA_ERR_INVALID_ARG;
    const spectra_trdc_layer &r = t->rec[i];
    void *dst[kBuffers] = {codes, scales, zeros, outlier_idx, outlier_w, bulk_idx};
    for (int b = 0; b < kBuffers; ++b) {
        if (r.bytes[b] == 0) continue;
        if (!dst[b]) return SPECTRA_ERR_INVALID_ARG;
        if (mem == SPECTRA_MEM_DEVICE && ((uintptr_t)dst[b] & (b == 3 ? 3u : 15u)))
            return SPECTRA_ERR_ALIGN;
    }
    if (mem == SPECTRA_MEM_DEVICE && !staging) return SPECTRA_ERR_INVALID_ARG;
    if (staging && staging_bytes < kMinStaging) return SPECTRA_ERR_BUFFER_TOO_SMALL;
    spectra_status st = SPECTRA_OK;
    {
        Halves h(mem == SPECTRA_MEM_DEVICE);
        if (!h.ok) st = SPECTRA_ERR_CUDA;
        const size_t half = (staging_bytes / 2) & ~(size_t)15;
        for (int b = 0; b < kBuffers && st == SPECTRA_OK; ++b) {
            if (r.bytes[b] == 0) continue;
            uint32_t c = 0;
            uint8_t *d = static_cast<uint8_t *>(dst[b]);
            uint8_t *stg = static_cast<uint8_t *>(staging);
            if (mem == SPECTRA_MEM_DEVICE) {
                DeviceCopier cp{h, (cudaStream_t)stream};
                st = load_buffer(t->fd, r.offset[b], r.bytes[b], d, stg, half, verify != 0, &c, cp);
            } else if (staging) {
                HostCopier cp;
                st = load_buffer(t->fd, r.offset[b], r.bytes[b], d, stg, half, verify != 0, &c, cp);
            } else {
                if (!pread_all(t->fd, d, (size_t)r.bytes[b], r.offset[b])) st = SPECTRA_ERR_IO;
                else if (verify) c = crc(0, d, (size_t)r.bytes[b]);
            }
            if (st == SPECTRA_OK && verify && c != r.crc32[b]) st = SPECTRA_ERR_FORMAT;
        }
    }
    if (st == SPECTRA_OK && layer_out) {
        const bool compact = (r.flags & 1u) != 0;
        layer_out->n = r.n;
        layer_out->k = r.k;
        layer_out->n_outliers = r.n_outliers;
        layer_out->codes = codes;
        layer_out->scales = scales;
        layer_out->zeros = zeros;
        layer_out->outlier_idx = r.n_outliers > 0 ? outlier_idx : nullptr;
        layer_out->outlier_w = r.n_outliers > 0 ? outlier_w : nullptr;
        layer_out->k_bulk = compact ? r.k_bulk : r.k;
        layer_out->bulk_idx = compact ? bulk_idx : nullptr;
    }
    return st;
}

void spectra_trdc_close(spectra_trdc *t) {
    if (!t) return;
    ::close(t->fd);
    std::free(t->rec);
    std::free(t);
}

}  // extern "C"

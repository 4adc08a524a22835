// wc_api.cu -- the extern "C" boundary of libwcodec: argument checks, layout
// arithmetic and kernel launches. Declarations and their contracts are in
// include/wcodec.h.
#include <stdint.h>
#include <string.h>

#include "../../include/wcodec.h"
#include "wc_internal.cuh"

namespace {

constexpr uint64_t kDefaultTimeoutNs = 1000000000ull;  // bounded look-back wait: 1 s

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool args_ok(uint64_t n, uint32_t block) { return wc::block_ok(block) && n <= wc::kMaxElems; }

int check_compress_args(const void* d_in, uint64_t n, uint32_t block, void* d_out,
                        uint64_t out_capacity, uint64_t* d_out_bytes, void* d_workspace,
                        uint64_t workspace_bytes, bool fp32 = false) {
    if (!args_ok(n, block) || d_out == nullptr || d_out_bytes == nullptr || d_workspace == nullptr ||
        (n > 0 && d_in == nullptr))
        return WC_ERR_INVALID_ARG;
    if ((n > 0 && !aligned16(d_in)) || !aligned16(d_out) || !aligned16(d_workspace) ||
        (reinterpret_cast<uintptr_t>(d_out_bytes) & 7u) != 0)
        return WC_ERR_INVALID_ARG;
    if (out_capacity < wc::bound_bytes(n, block, fp32) ||
        workspace_bytes < wc::encode_workspace_bytes(wc::encode_tiles(n)))
        return WC_ERR_BUFFER_TOO_SMALL;
    return WC_OK;
}

wc::EncodeItem to_encode_item(const void* d_in, uint64_t n, uint32_t block, void* d_out,
                              uint64_t* d_out_bytes) {
    wc::EncodeItem e;
    e.in = static_cast<const uint16_t*>(d_in);
    e.out = static_cast<uint8_t*>(d_out);
    e.out_bytes = d_out_bytes;
    e.n = n;
    e.block = block;
    e.reserved = 0;
    return e;
}

// Workspace of a batch: one part per launch of up to WC_BATCH_MAX tensors.
uint64_t batch_workspace_bytes(const wc_compress_item* items, uint32_t count) {
    uint64_t total = 0;
    for (uint32_t base = 0; base < count; base += WC_BATCH_MAX) {
        const uint32_t c = (count - base < WC_BATCH_MAX) ? count - base : WC_BATCH_MAX;
        uint64_t tiles = 0;
        for (uint32_t i = 0; i < c; ++i) tiles += wc::encode_tiles(items[base + i].n);
        total += (wc::encode_workspace_bytes(tiles) + 15) & ~uint64_t(15);
    }
    return total;
}

int check_decode_item(const wc_batch_item& it, bool fp32 = false) {
    if (!args_ok(it.n, it.block) || it.stream == nullptr || (it.n > 0 && it.out == nullptr) ||
        it.reserved != 0)
        return WC_ERR_INVALID_ARG;
    if (!aligned16(it.stream) || (it.n > 0 && !aligned16(it.out))) return WC_ERR_INVALID_ARG;
    // the fixed sections alone need off_exp bytes
    if (it.stream_bytes < wc::make_layout(it.n, it.block, fp32).off_exp) return WC_ERR_CORRUPT_STREAM;
    return WC_OK;
}

wc::DecodeItem to_item(const wc_batch_item& it) {
    wc::DecodeItem d;
    d.stream = static_cast<const uint8_t*>(it.stream);
    d.stream_bytes = it.stream_bytes;
    d.out = static_cast<uint16_t*>(it.out);
    d.n = it.n;
    d.block = it.block;
    d.reserved = 0;
    return d;
}

uint64_t get_le(const uint8_t* p, int nbytes) {
    uint64_t v = 0;
    for (int k = 0; k < nbytes; ++k) v |= uint64_t(p[k]) << (8 * k);
    return v;
}

}  // namespace

extern "C" {

uint64_t wc_bound(uint64_t n, uint32_t block) {
    return args_ok(n, block) ? wc::bound_bytes(n, block) : 0;
}

uint64_t wc_workspace_size(uint64_t n, uint32_t block) {
    return args_ok(n, block) ? wc::encode_workspace_bytes(wc::encode_tiles(n)) : 0;
}

static int compress_impl(const void* d_in, uint64_t n, uint32_t block, void* d_out,
                         uint64_t out_capacity, uint64_t* d_out_bytes, void* d_workspace,
                         uint64_t workspace_bytes, int32_t* d_status, uint64_t timeout_ns,
                         uint32_t first_ticket, void* stream) {
    const int rc = check_compress_args(d_in, n, block, d_out, out_capacity, d_out_bytes,
                                       d_workspace, workspace_bytes);
    if (rc != WC_OK) return rc;
    const wc::EncodeItem item = to_encode_item(d_in, n, block, d_out, d_out_bytes);
    const cudaError_t err = wc::launch_encode(&item, 1, d_workspace, d_status, timeout_ns,
                                              first_ticket, static_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? WC_OK : WC_ERR_CUDA;
}

int wc_compress(const void* d_in, uint64_t n, uint32_t block, void* d_out, uint64_t out_capacity,
                uint64_t* d_out_bytes, void* d_workspace, uint64_t workspace_bytes,
                int32_t* d_status, void* stream) {
    return compress_impl(d_in, n, block, d_out, out_capacity, d_out_bytes, d_workspace,
                         workspace_bytes, d_status, kDefaultTimeoutNs, 0, stream);
}

int wc_debug_compress_stalled(const void* d_in, uint64_t n, uint32_t block, void* d_out,
                              uint64_t out_capacity, uint64_t* d_out_bytes, void* d_workspace,
                              uint64_t workspace_bytes, int32_t* d_status, uint64_t timeout_ns,
                              void* stream) {
    if (wc::num_tiles(n) < 2 || timeout_ns == 0 || timeout_ns > 10 * kDefaultTimeoutNs)
        return WC_ERR_INVALID_ARG;
    return compress_impl(d_in, n, block, d_out, out_capacity, d_out_bytes, d_workspace,
                         workspace_bytes, d_status, timeout_ns, 1, stream);
}

int wc_compress_noalloc(const void* d_in, uint64_t n, uint32_t block, void* d_out,
                        uint64_t out_capacity, uint64_t* d_out_bytes, int32_t* d_status,
                        void* stream) {
    // Size first: nothing is looked up or enqueued for a tensor the array cannot serve.
    if (n > wc::noalloc_max_elems()) return WC_ERR_BUFFER_TOO_SMALL;
    if (!wc::block_ok(block) || d_out == nullptr || d_out_bytes == nullptr ||
        (n > 0 && d_in == nullptr))
        return WC_ERR_INVALID_ARG;
    if ((n > 0 && !aligned16(d_in)) || !aligned16(d_out) ||
        (reinterpret_cast<uintptr_t>(d_out_bytes) & 7u) != 0)
        return WC_ERR_INVALID_ARG;
    if (out_capacity < wc::bound_bytes(n, block)) return WC_ERR_BUFFER_TOO_SMALL;
    void* scratch = nullptr;
    uint64_t scratch_bytes = 0;
    if (wc::noalloc_scratch(&scratch, &scratch_bytes) != cudaSuccess) return WC_ERR_CUDA;
    if (scratch_bytes < wc::encode_workspace_bytes(wc::encode_tiles(n)))
        return WC_ERR_BUFFER_TOO_SMALL;
    const wc::EncodeItem item = to_encode_item(d_in, n, block, d_out, d_out_bytes);
    const cudaError_t err = wc::launch_encode(&item, 1, scratch, d_status, kDefaultTimeoutNs, 0,
                                              static_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? WC_OK : WC_ERR_CUDA;
}

uint64_t wc_compress_batch_workspace_size(const wc_compress_item* h_items, uint32_t count) {
    if (h_items == nullptr && count > 0) return 0;
    for (uint32_t i = 0; i < count; ++i)
        if (!args_ok(h_items[i].n, h_items[i].block)) return 0;
    return batch_workspace_bytes(h_items, count);
}

int wc_compress_batch(const wc_compress_item* h_items, uint32_t count, void* d_workspace,
                      uint64_t workspace_bytes, int32_t* d_status, void* stream) {
    if (h_items == nullptr && count > 0) return WC_ERR_INVALID_ARG;
    if (count == 0) return WC_OK;
    for (uint32_t i = 0; i < count; ++i) {  // check everything before launching anything
        const wc_compress_item& it = h_items[i];
        if (it.reserved != 0) return WC_ERR_INVALID_ARG;
        const int rc = check_compress_args(it.in, it.n, it.block, it.out, it.out_capacity,
                                           it.out_bytes, d_workspace, UINT64_MAX);
        if (rc != WC_OK) return rc;
    }
    if (workspace_bytes < batch_workspace_bytes(h_items, count)) return WC_ERR_BUFFER_TOO_SMALL;
    wc::EncodeItem chunk[WC_BATCH_MAX];
    uint8_t* ws = static_cast<uint8_t*>(d_workspace);
    for (uint32_t base = 0; base < count; base += WC_BATCH_MAX) {
        const uint32_t c = (count - base < WC_BATCH_MAX) ? count - base : WC_BATCH_MAX;
        for (uint32_t i = 0; i < c; ++i) {
            const wc_compress_item& it = h_items[base + i];
            chunk[i] = to_encode_item(it.in, it.n, it.block, it.out, it.out_bytes);
        }
        const cudaError_t err = wc::launch_encode(chunk, c, ws, d_status, kDefaultTimeoutNs, 0,
                                                  static_cast<cudaStream_t>(stream));
        if (err != cudaSuccess) return WC_ERR_CUDA;
        ws += batch_workspace_bytes(h_items + base, c);
    }
    return WC_OK;
}

int wc_decompress(const void* d_stream, uint64_t stream_bytes, void* d_out, uint64_t n,
                  uint32_t block, int32_t* d_status, void* stream) {
    wc_batch_item it;
    it.stream = d_stream;
    it.stream_bytes = stream_bytes;
    it.out = d_out;
    it.n = n;
    it.block = block;
    it.reserved = 0;
    const int rc = check_decode_item(it);
    if (rc != WC_OK) return rc;
    const wc::DecodeItem d = to_item(it);
    const cudaError_t err = wc::launch_decode(&d, 1, d_status, static_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? WC_OK : WC_ERR_CUDA;
}

uint64_t wc_bound_fp32(uint64_t n, uint32_t block) {
    return args_ok(n, block) ? wc::bound_bytes(n, block, true) : 0;
}

int wc_compress_fp32(const void* d_in, uint64_t n, uint32_t block, void* d_out,
                     uint64_t out_capacity, uint64_t* d_out_bytes, void* d_workspace,
                     uint64_t workspace_bytes, int32_t* d_status, void* stream) {
    const int rc = check_compress_args(d_in, n, block, d_out, out_capacity, d_out_bytes,
                                       d_workspace, workspace_bytes, true);
    if (rc != WC_OK) return rc;
    const wc::EncodeItem item = to_encode_item(d_in, n, block, d_out, d_out_bytes);
    const cudaError_t err = wc::launch_encode(&item, 1, d_workspace, d_status, kDefaultTimeoutNs,
                                              0, static_cast<cudaStream_t>(stream), true);
    return err == cudaSuccess ? WC_OK : WC_ERR_CUDA;
}

int wc_decompress_fp32(const void* d_stream, uint64_t stream_bytes, void* d_out, uint64_t n,
                       uint32_t block, int32_t* d_status, void* stream) {
    wc_batch_item it;
    it.stream = d_stream;
    it.stream_bytes = stream_bytes;
    it.out = d_out;
    it.n = n;
    it.block = block;
    it.reserved = 0;
    const int rc = check_decode_item(it, true);
    if (rc != WC_OK) return rc;
    const wc::DecodeItem d = to_item(it);
    const cudaError_t err =
        wc::launch_decode(&d, 1, d_status, static_cast<cudaStream_t>(stream), wc::kKindF32);
    return err == cudaSuccess ? WC_OK : WC_ERR_CUDA;
}

int wc_decompress_batch(const wc_batch_item* h_items, uint32_t count, int32_t* d_status,
                        void* stream) {
    if (h_items == nullptr && count > 0) return WC_ERR_INVALID_ARG;
    for (uint32_t i = 0; i < count; ++i) {  // validate everything before launching anything
        const int rc = check_decode_item(h_items[i]);
        if (rc != WC_OK) return rc;
    }
    wc::DecodeItem chunk[WC_BATCH_MAX];
    for (uint32_t base = 0; base < count; base += WC_BATCH_MAX) {
        const uint32_t c = (count - base < WC_BATCH_MAX) ? count - base : WC_BATCH_MAX;
        for (uint32_t i = 0; i < c; ++i) chunk[i] = to_item(h_items[base + i]);
        const cudaError_t err =
            wc::launch_decode(chunk, c, d_status, static_cast<cudaStream_t>(stream));
        if (err != cudaSuccess) return WC_ERR_CUDA;
    }
    return WC_OK;
}

uint64_t wc_bound_escape(uint64_t n, uint32_t block) {
    return args_ok(n, block) ? wc::bound_bytes_escape(n, block) : 0;
}

uint64_t wc_workspace_size_escape(uint64_t n, uint32_t block) {
    if (!args_ok(n, block)) return 0;
    const wc::EncodeItem item = to_encode_item(nullptr, n, block, nullptr, nullptr);
    return wc::escape_workspace_bytes(&item, 1);
}

static int check_escape_item(const void* d_in, uint64_t n, uint32_t block, const void* d_out,
                             uint64_t out_capacity, const uint64_t* d_out_bytes) {
    if (!args_ok(n, block) || d_out == nullptr || d_out_bytes == nullptr ||
        (n > 0 && d_in == nullptr))
        return WC_ERR_INVALID_ARG;
    if ((n > 0 && !aligned16(d_in)) || !aligned16(d_out) ||
        (reinterpret_cast<uintptr_t>(d_out_bytes) & 7u) != 0)
        return WC_ERR_INVALID_ARG;
    if (out_capacity < wc::bound_bytes_escape(n, block)) return WC_ERR_BUFFER_TOO_SMALL;
    return WC_OK;
}

int wc_compress_escape(const void* d_in, uint64_t n, uint32_t block, void* d_out,
                       uint64_t out_capacity, uint64_t* d_out_bytes, void* d_workspace,
                       uint64_t workspace_bytes, int32_t* d_status, void* stream) {
    (void)d_status;  // nothing in these kernels waits, so nothing can time out
    const int rc = check_escape_item(d_in, n, block, d_out, out_capacity, d_out_bytes);
    if (rc != WC_OK) return rc;
    if (d_workspace == nullptr || !aligned16(d_workspace)) return WC_ERR_INVALID_ARG;
    const wc::EncodeItem item = to_encode_item(d_in, n, block, d_out, d_out_bytes);
    if (workspace_bytes < wc::escape_workspace_bytes(&item, 1)) return WC_ERR_BUFFER_TOO_SMALL;
    const cudaError_t err =
        wc::launch_encode_escape(&item, 1, d_workspace, static_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? WC_OK : WC_ERR_CUDA;
}

// Host-side copies of a batch's items (at most this many per call of the helpers below).
static uint64_t escape_batch_workspace(const wc_compress_item* h_items, uint32_t count) {
    uint64_t total = 0;
    wc::EncodeItem chunk[WC_BATCH_MAX];
    for (uint32_t base = 0; base < count; base += WC_BATCH_MAX) {
        const uint32_t c = (count - base < WC_BATCH_MAX) ? count - base : WC_BATCH_MAX;
        for (uint32_t i = 0; i < c; ++i) {
            const wc_compress_item& it = h_items[base + i];
            chunk[i] = to_encode_item(it.in, it.n, it.block, it.out, it.out_bytes);
        }
        total += wc::escape_workspace_bytes(chunk, c);
    }
    return total;
}

uint64_t wc_compress_escape_batch_workspace_size(const wc_compress_item* h_items, uint32_t count) {
    if (h_items == nullptr && count > 0) return 0;
    for (uint32_t i = 0; i < count; ++i)
        if (!args_ok(h_items[i].n, h_items[i].block)) return 0;
    return escape_batch_workspace(h_items, count);
}

int wc_compress_escape_batch(const wc_compress_item* h_items, uint32_t count, void* d_workspace,
                             uint64_t workspace_bytes, int32_t* d_status, void* stream) {
    (void)d_status;
    if (h_items == nullptr && count > 0) return WC_ERR_INVALID_ARG;
    if (count == 0) return WC_OK;
    for (uint32_t i = 0; i < count; ++i) {  // check everything before launching anything
        const wc_compress_item& it = h_items[i];
        if (it.reserved != 0) return WC_ERR_INVALID_ARG;
        const int rc = check_escape_item(it.in, it.n, it.block, it.out, it.out_capacity,
                                         it.out_bytes);
        if (rc != WC_OK) return rc;
    }
    if (d_workspace == nullptr || !aligned16(d_workspace)) return WC_ERR_INVALID_ARG;
    if (workspace_bytes < escape_batch_workspace(h_items, count)) return WC_ERR_BUFFER_TOO_SMALL;
    wc::EncodeItem chunk[WC_BATCH_MAX];
    uint8_t* ws = static_cast<uint8_t*>(d_workspace);
    for (uint32_t base = 0; base < count; base += WC_BATCH_MAX) {
        const uint32_t c = (count - base < WC_BATCH_MAX) ? count - base : WC_BATCH_MAX;
        for (uint32_t i = 0; i < c; ++i) {
            const wc_compress_item& it = h_items[base + i];
            chunk[i] = to_encode_item(it.in, it.n, it.block, it.out, it.out_bytes);
        }
        const cudaError_t err =
            wc::launch_encode_escape(chunk, c, ws, static_cast<cudaStream_t>(stream));
        if (err != cudaSuccess) return WC_ERR_CUDA;
        ws += wc::escape_workspace_bytes(chunk, c);
    }
    return WC_OK;
}

int wc_decompress_escape(const void* d_stream, uint64_t stream_bytes, void* d_out, uint64_t n,
                         uint32_t block, int32_t* d_status, void* stream) {
    wc_batch_item it;
    it.stream = d_stream;
    it.stream_bytes = stream_bytes;
    it.out = d_out;
    it.n = n;
    it.block = block;
    it.reserved = 0;
    return wc_decompress_escape_batch(&it, 1, d_status, stream);
}

int wc_decompress_escape_batch(const wc_batch_item* h_items, uint32_t count, int32_t* d_status,
                               void* stream) {
    if (h_items == nullptr && count > 0) return WC_ERR_INVALID_ARG;
    for (uint32_t i = 0; i < count; ++i) {  // validate everything before launching anything
        const int rc = check_decode_item(h_items[i]);
        if (rc != WC_OK) return rc;
    }
    wc::DecodeItem chunk[WC_BATCH_MAX];
    for (uint32_t base = 0; base < count; base += WC_BATCH_MAX) {
        const uint32_t c = (count - base < WC_BATCH_MAX) ? count - base : WC_BATCH_MAX;
        for (uint32_t i = 0; i < c; ++i) chunk[i] = to_item(h_items[base + i]);
        const cudaError_t err = wc::launch_decode(chunk, c, d_status,
                                                  static_cast<cudaStream_t>(stream), wc::kKindEscape);
        if (err != cudaSuccess) return WC_ERR_CUDA;
    }
    return WC_OK;
}

static int check_tans_item(const wc_batch_item& it) {
    if (!wc::tans_chunk_ok(it.block) || it.n > wc::kMaxElems || it.stream == nullptr ||
        (it.n > 0 && it.out == nullptr) || it.reserved != 0)
        return WC_ERR_INVALID_ARG;
    if (!aligned16(it.stream) || (it.n > 0 && !aligned16(it.out))) return WC_ERR_INVALID_ARG;
    if (it.stream_bytes < wc::tans_fixed_bytes(it.n, it.block)) return WC_ERR_CORRUPT_STREAM;
    return WC_OK;
}

uint64_t wc_bound_tans(uint64_t n, uint32_t chunk, uint32_t table_log) {
    if (!wc::tans_chunk_ok(chunk) || table_log < 8 || table_log > 12 || n > wc::kMaxElems) return 0;
    return wc::tans_bound_bytes(n, chunk, table_log);
}

static int tans_encode_items(const wc_compress_item* h_items, uint32_t count, uint32_t table_log,
                             wc::EncodeItem* items) {
    if (table_log < 8 || table_log > 12) return WC_ERR_INVALID_ARG;
    for (uint32_t i = 0; i < count; ++i) {
        const wc_compress_item& it = h_items[i];
        if (!wc::tans_chunk_ok(it.block) || it.n > wc::kMaxElems || it.out == nullptr ||
            it.out_bytes == nullptr || (it.n > 0 && it.in == nullptr) || it.reserved != 0)
            return WC_ERR_INVALID_ARG;
        if ((it.n > 0 && !aligned16(it.in)) || !aligned16(it.out) ||
            (reinterpret_cast<uintptr_t>(it.out_bytes) & 7u) != 0)
            return WC_ERR_INVALID_ARG;
        if (it.out_capacity < wc::tans_bound_bytes(it.n, it.block, table_log))
            return WC_ERR_BUFFER_TOO_SMALL;
        items[i] = to_encode_item(it.in, it.n, it.block, it.out, it.out_bytes);
    }
    return WC_OK;
}

uint64_t wc_compress_tans_batch_workspace_size(const wc_compress_item* h_items, uint32_t count) {
    if (h_items == nullptr && count > 0) return 0;
    uint64_t total = 0;
    for (uint32_t base = 0; base < count; base += WC_BATCH_MAX) {
        const uint32_t c = (count - base < WC_BATCH_MAX) ? count - base : WC_BATCH_MAX;
        wc::EncodeItem items[WC_BATCH_MAX];
        for (uint32_t i = 0; i < c; ++i) {
            items[i].n = h_items[base + i].n;
            items[i].block = wc::tans_chunk_ok(h_items[base + i].block) ? h_items[base + i].block : 1024u;
        }
        total += wc::tans_workspace_bytes(items, c);
    }
    return total;
}

int wc_compress_tans_batch(const wc_compress_item* h_items, uint32_t count, uint32_t table_log,
                           void* d_workspace, uint64_t workspace_bytes, void* stream) {
    if ((h_items == nullptr && count > 0) || (count > 0 && d_workspace == nullptr) ||
        (count > 0 && !aligned16(d_workspace)))
        return WC_ERR_INVALID_ARG;
    if (workspace_bytes < wc_compress_tans_batch_workspace_size(h_items, count))
        return WC_ERR_BUFFER_TOO_SMALL;
    uint8_t* ws = static_cast<uint8_t*>(d_workspace);
    for (uint32_t base = 0; base < count; base += WC_BATCH_MAX) {
        const uint32_t c = (count - base < WC_BATCH_MAX) ? count - base : WC_BATCH_MAX;
        wc::EncodeItem items[WC_BATCH_MAX];
        uint32_t logs[WC_BATCH_MAX];
        const int rc = tans_encode_items(h_items + base, c, table_log, items);
        if (rc != WC_OK) return rc;
        for (uint32_t i = 0; i < c; ++i) logs[i] = table_log;
        const cudaError_t err =
            wc::launch_encode_tans(items, logs, c, ws, static_cast<cudaStream_t>(stream));
        if (err != cudaSuccess) return WC_ERR_CUDA;
        ws += wc::tans_workspace_bytes(items, c);
    }
    return WC_OK;
}

int wc_compress_tans(const void* d_in, uint64_t n, uint32_t chunk, uint32_t table_log, void* d_out,
                     uint64_t out_capacity, uint64_t* d_out_bytes, void* d_workspace,
                     uint64_t workspace_bytes, void* stream) {
    wc_compress_item it;
    it.in = d_in;
    it.n = n;
    it.block = chunk;
    it.reserved = 0;
    it.out = d_out;
    it.out_capacity = out_capacity;
    it.out_bytes = d_out_bytes;
    return wc_compress_tans_batch(&it, 1, table_log, d_workspace, workspace_bytes, stream);
}

int wc_decompress_tans_batch(const wc_batch_item* h_items, uint32_t count, int32_t* d_status,
                             void* stream) {
    if (h_items == nullptr && count > 0) return WC_ERR_INVALID_ARG;
    for (uint32_t i = 0; i < count; ++i) {  // validate everything before launching anything
        const int rc = check_tans_item(h_items[i]);
        if (rc != WC_OK) return rc;
    }
    wc::DecodeItem chunk[WC_BATCH_MAX];
    for (uint32_t base = 0; base < count; base += WC_BATCH_MAX) {
        const uint32_t c = (count - base < WC_BATCH_MAX) ? count - base : WC_BATCH_MAX;
        for (uint32_t i = 0; i < c; ++i) chunk[i] = to_item(h_items[base + i]);
        const cudaError_t err =
            wc::launch_decode_tans(chunk, c, d_status, static_cast<cudaStream_t>(stream));
        if (err != cudaSuccess) return WC_ERR_CUDA;
    }
    return WC_OK;
}

int wc_decompress_tans(const void* d_stream, uint64_t stream_bytes, void* d_out, uint64_t n,
                       uint32_t chunk, int32_t* d_status, void* stream) {
    wc_batch_item it;
    it.stream = d_stream;
    it.stream_bytes = stream_bytes;
    it.out = d_out;
    it.n = n;
    it.block = chunk;
    it.reserved = 0;
    return wc_decompress_tans_batch(&it, 1, d_status, stream);
}

// The device's address of page-locked host memory (cudaHostAlloc, cudaMallocHost
// or cudaHostRegister); nullptr for any other pointer. A host-side query: it
// neither allocates nor synchronizes.
static const void* mapped_host_address(const void* h) {
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, h) != cudaSuccess) {
        (void)cudaGetLastError();  // a failed query leaves a (non-sticky) error: clear it
        return nullptr;
    }
    return a.type == cudaMemoryTypeHost ? a.devicePointer : nullptr;
}

int wc_decompress_host_batch(const wc_batch_item* h_items, uint32_t count, uint32_t flags,
                             int32_t* d_status, void* stream) {
    if ((h_items == nullptr && count > 0) || (flags != 0u && flags != WC_FLAG_ESCAPE))
        return WC_ERR_INVALID_ARG;
    for (uint32_t i = 0; i < count; ++i) {  // validate everything before launching anything
        const int rc = check_decode_item(h_items[i]);
        if (rc != WC_OK) return rc;
        const void* dev = mapped_host_address(h_items[i].stream);
        if (dev == nullptr || !aligned16(dev)) return WC_ERR_INVALID_ARG;
    }
    const int kind = flags == WC_FLAG_ESCAPE ? wc::kKindEscape : wc::kKindPlain;
    wc::DecodeItem chunk[WC_BATCH_MAX];
    for (uint32_t base = 0; base < count; base += WC_BATCH_MAX) {
        const uint32_t c = (count - base < WC_BATCH_MAX) ? count - base : WC_BATCH_MAX;
        for (uint32_t i = 0; i < c; ++i) {
            chunk[i] = to_item(h_items[base + i]);
            chunk[i].stream = static_cast<const uint8_t*>(mapped_host_address(h_items[base + i].stream));
        }
        const cudaError_t err = wc::launch_decode(chunk, c, d_status,
                                                  static_cast<cudaStream_t>(stream), kind, true);
        if (err != cudaSuccess) return WC_ERR_CUDA;
    }
    return WC_OK;
}

int wc_decompress_host(const void* h_stream, uint64_t stream_bytes, void* d_out, uint64_t n,
                       uint32_t block, uint32_t flags, int32_t* d_status, void* stream) {
    wc_batch_item it;
    it.stream = h_stream;
    it.stream_bytes = stream_bytes;
    it.out = d_out;
    it.n = n;
    it.block = block;
    it.reserved = 0;
    return wc_decompress_host_batch(&it, 1, flags, d_status, stream);
}

static int check_gemv_item(const wc_gemv_item& it, uint32_t n_vec) {
    if (n_vec != 1 && n_vec != 2 && n_vec != 4) return WC_ERR_INVALID_ARG;
    if (!wc::block_ok(it.block) || it.reserved != 0 || it.stream == nullptr ||
        (it.rows > 0 && (it.x == nullptr || it.y == nullptr)) || it.cols == 0 ||
        it.cols % it.block != 0 || uint64_t(it.rows) * it.cols > wc::kMaxElems)
        return WC_ERR_INVALID_ARG;
    if (!aligned16(it.stream) || !aligned16(it.x) || (reinterpret_cast<uintptr_t>(it.y) & 3u) != 0)
        return WC_ERR_INVALID_ARG;
    if (it.stream_bytes < wc::make_layout(uint64_t(it.rows) * it.cols, it.block).off_exp)
        return WC_ERR_CORRUPT_STREAM;
    return WC_OK;
}

static wc::GemvItem to_gemv_item(const wc_gemv_item& it) {
    wc::GemvItem g;
    g.stream = static_cast<const uint8_t*>(it.stream);
    g.stream_bytes = it.stream_bytes;
    g.x = static_cast<const uint16_t*>(it.x);
    g.y = it.y;
    g.rows = it.rows;
    g.cols = it.cols;
    g.block = it.block;
    g.reserved = 0;
    return g;
}

int wc_gemv(const void* d_stream, uint64_t stream_bytes, uint32_t rows, uint32_t cols,
            uint32_t block, const void* d_x, uint32_t n_vec, float* d_y, int32_t* d_status,
            void* stream) {
    wc_gemv_item it;
    it.stream = d_stream;
    it.stream_bytes = stream_bytes;
    it.x = d_x;
    it.y = d_y;
    it.rows = rows;
    it.cols = cols;
    it.block = block;
    it.reserved = 0;
    return wc_gemv_batch(&it, 1, n_vec, d_status, stream);
}

int wc_gemv_batch(const wc_gemv_item* h_items, uint32_t count, uint32_t n_vec, int32_t* d_status,
                  void* stream) {
    if (h_items == nullptr && count > 0) return WC_ERR_INVALID_ARG;
    for (uint32_t i = 0; i < count; ++i) {  // check everything before launching anything
        const int rc = check_gemv_item(h_items[i], n_vec);
        if (rc != WC_OK) return rc;
    }
    wc::GemvItem chunk[256];
    for (uint32_t base = 0; base < count; base += 256) {
        const uint32_t c = (count - base < 256) ? count - base : 256;
        for (uint32_t i = 0; i < c; ++i) chunk[i] = to_gemv_item(h_items[base + i]);
        const cudaError_t err =
            wc::launch_gemv(chunk, c, n_vec, d_status, static_cast<cudaStream_t>(stream));
        if (err != cudaSuccess) return WC_ERR_CUDA;
    }
    return WC_OK;
}

static int check_gemm_item(const wc_gemv_item& it, uint32_t tokens, bool escape) {
    if (tokens < 1 || tokens > WC_GEMM_MAX_TOKENS) return WC_ERR_INVALID_ARG;
    if (!wc::block_ok(it.block) || it.reserved != 0 || it.stream == nullptr ||
        (it.rows > 0 && (it.x == nullptr || it.y == nullptr)) || it.cols == 0 ||
        it.cols % 128u != 0 || uint64_t(it.rows) * it.cols > wc::kMaxElems)
        return WC_ERR_INVALID_ARG;
    if (escape && it.cols % it.block != 0) return WC_ERR_INVALID_ARG;  // rows of whole blocks
    if (!aligned16(it.stream) || !aligned16(it.x) || (reinterpret_cast<uintptr_t>(it.y) & 3u) != 0)
        return WC_ERR_INVALID_ARG;
    if (it.stream_bytes < wc::make_layout(uint64_t(it.rows) * it.cols, it.block).off_exp)
        return WC_ERR_CORRUPT_STREAM;
    return WC_OK;
}

int wc_gemm(const void* d_stream, uint64_t stream_bytes, uint32_t rows, uint32_t cols,
            uint32_t block, const void* d_x, uint32_t tokens, float* d_y, int32_t* d_status,
            void* stream) {
    wc_gemv_item it;
    it.stream = d_stream;
    it.stream_bytes = stream_bytes;
    it.x = d_x;
    it.y = d_y;
    it.rows = rows;
    it.cols = cols;
    it.block = block;
    it.reserved = 0;
    return wc_gemm_batch(&it, 1, tokens, d_status, stream);
}

int wc_gemm_batch(const wc_gemv_item* h_items, uint32_t count, uint32_t tokens, int32_t* d_status,
                  void* stream) {
    return wc_gemm_batch_flags(h_items, count, tokens, 0, d_status, stream);
}

int wc_gemm_batch_flags(const wc_gemv_item* h_items, uint32_t count, uint32_t tokens,
                        uint32_t flags, int32_t* d_status, void* stream) {
    if (h_items == nullptr && count > 0) return WC_ERR_INVALID_ARG;
    if (flags != 0 && flags != WC_FLAG_ESCAPE) return WC_ERR_INVALID_ARG;
    const bool escape = flags == WC_FLAG_ESCAPE;
    for (uint32_t i = 0; i < count; ++i) {  // check everything before launching anything
        const int rc = check_gemm_item(h_items[i], tokens, escape);
        if (rc != WC_OK) return rc;
    }
    constexpr uint32_t kChunk = wc::kGemmBatchMax;
    wc::GemvItem chunk[kChunk];
    for (uint32_t base = 0; base < count; base += kChunk) {
        const uint32_t c = (count - base < kChunk) ? count - base : kChunk;
        for (uint32_t i = 0; i < c; ++i) chunk[i] = to_gemv_item(h_items[base + i]);
        const cudaError_t err =
            wc::launch_gemm(chunk, c, tokens, escape, d_status, static_cast<cudaStream_t>(stream));
        if (err != cudaSuccess) return WC_ERR_CUDA;
    }
    return WC_OK;
}

int wc_stream_info(const void* h_header, uint64_t header_bytes, uint64_t* n, uint32_t* block,
                   uint64_t* total_bytes) {
    if (h_header == nullptr || header_bytes < WC_HEADER_BYTES) return WC_ERR_INVALID_ARG;
    const uint8_t* p = static_cast<const uint8_t*>(h_header);
    const uint64_t nn = get_le(p + 16, 8);
    const uint32_t B = uint32_t(get_le(p + 8, 4));
    const uint64_t flags = get_le(p + 12, 4);
    if (get_le(p, 4) != wc::kMagic || get_le(p + 4, 2) != wc::kVersion ||
        get_le(p + 6, 2) != wc::kHeaderBytes)
        return WC_ERR_CORRUPT_STREAM;
    if (flags == 4) {  // tANS-coded: chunk size in the block field, table log at 88
        const uint64_t R = get_le(p + 88, 4);
        const uint64_t E = get_le(p + 64, 8), total = get_le(p + 72, 8);
        if (!wc::tans_chunk_ok(B) || nn > wc::kMaxElems || R < 8 || R > 12 ||
            get_le(p + 24, 8) != (nn + B - 1) / B || get_le(p + 32, 8) != WC_HEADER_BYTES ||
            total != wc::tans_fixed_bytes(nn, B) + E || get_le(p + 56, 8) != wc::tans_fixed_bytes(nn, B) ||
            get_le(p + 80, 8) != 0)
            return WC_ERR_CORRUPT_STREAM;
        for (int k = 92; k < 128; ++k)
            if (p[k] != 0) return WC_ERR_CORRUPT_STREAM;
        if (n) *n = nn;
        if (block) *block = B;
        if (total_bytes) *total_bytes = total;
        return WC_OK;
    }
    if (flags > 2 || !args_ok(nn, B)) return WC_ERR_CORRUPT_STREAM;
    const wc::Layout L = wc::make_layout(nn, B, flags == 1);  // escape-coded: the BF16 layout
    const uint64_t E = get_le(p + 64, 8), total = get_le(p + 72, 8);
    if (get_le(p + 24, 8) != L.nb || get_le(p + 32, 8) != L.off_hdr ||
        get_le(p + 40, 8) != L.off_offs || get_le(p + 48, 8) != L.off_man ||
        get_le(p + 56, 8) != L.off_exp || E > nn + 16 || total != L.off_exp + E)
        return WC_ERR_CORRUPT_STREAM;
    if (get_le(p + 80, 8) != L.off_low) return WC_ERR_CORRUPT_STREAM;
    for (int k = 88; k < 128; ++k)
        if (p[k] != 0) return WC_ERR_CORRUPT_STREAM;
    if (n) *n = nn;
    if (block) *block = B;
    if (total_bytes) *total_bytes = total;
    return WC_OK;
}

const char* wc_status_string(int status) {
    switch (status) {
        case WC_OK: return "ok";
        case WC_ERR_INVALID_ARG: return "invalid argument";
        case WC_ERR_BUFFER_TOO_SMALL: return "buffer too small";
        case WC_ERR_CORRUPT_STREAM: return "corrupt stream";
        case WC_ERR_CUDA: return "CUDA error";
        case WC_ERR_TIMEOUT: return "in-kernel wait timed out";
        default: return "unknown status";
    }
}

}  // extern "C"

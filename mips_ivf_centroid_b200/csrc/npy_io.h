// NumPy .npy files (format versions 1.0 and 2.0) for the index directory:
// a header naming dtype, order and shape, then the array's bytes in C order.
// Host code only.
#pragma once

#include <cstdint>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

namespace ah {
namespace npy {

struct Header {
    std::string descr;              // e.g. "<f4", "<i8", "|u1", "<u2"
    std::vector<int64_t> shape;
    int64_t data_offset = 0;        // bytes before the array data
    int64_t file_bytes = 0;
};

inline int64_t item_size(const std::string& descr) {
    if (descr.size() < 3) return 0;
    const char kind = descr[1];
    if (kind != 'f' && kind != 'i' && kind != 'u') return 0;
    return std::atoi(descr.c_str() + 2);
}

inline int64_t count(const std::vector<int64_t>& shape) {
    int64_t c = 1;
    for (int64_t s : shape) c *= s;
    return c;
}

// Header text for `descr` and `shape`, padded with spaces and ended by '\n'
// so that the data starts at a multiple of 64 bytes (version 1.0).
inline std::string make_header(const std::string& descr, const std::vector<int64_t>& shape) {
    std::string d = "{'descr': '" + descr + "', 'fortran_order': False, 'shape': (";
    for (size_t i = 0; i < shape.size(); ++i) {
        d += std::to_string(shape[i]);
        d += (shape.size() == 1) ? "," : (i + 1 < shape.size() ? ", " : "");
    }
    d += "), }";
    const size_t pre = 10;                              // magic(6) + version(2) + length(2)
    size_t total = pre + d.size() + 1;
    const size_t pad = (64 - total % 64) % 64;
    d.append(pad, ' ');
    d += '\n';
    std::string out("\x93NUMPY\x01\x00", 8);
    const uint16_t len = static_cast<uint16_t>(d.size());
    out += static_cast<char>(len & 0xFF);
    out += static_cast<char>(len >> 8);
    out += d;
    return out;
}

// Value text after `key` in the header dict ("'key': value"), or "" if absent.
inline std::string dict_value(const std::string& h, const std::string& key) {
    const std::string k = "'" + key + "'";
    size_t p = h.find(k);
    if (p == std::string::npos) return "";
    p = h.find(':', p + k.size());
    if (p == std::string::npos) return "";
    ++p;
    while (p < h.size() && h[p] == ' ') ++p;
    if (p >= h.size()) return "";
    if (h[p] == '\'') {
        const size_t e = h.find('\'', p + 1);
        return e == std::string::npos ? "" : h.substr(p, e - p + 1);
    }
    if (h[p] == '(') {
        const size_t e = h.find(')', p);
        return e == std::string::npos ? "" : h.substr(p, e - p + 1);
    }
    size_t e = p;
    while (e < h.size() && h[e] != ',' && h[e] != '}') ++e;
    return h.substr(p, e - p);
}

// Parses the header of `path`; returns "" on success or what is wrong.
inline std::string read_header(const char* path, Header* out) {
    FILE* f = std::fopen(path, "rb");
    if (!f) return "cannot open";
    std::fseek(f, 0, SEEK_END);
    out->file_bytes = std::ftell(f);
    std::fseek(f, 0, SEEK_SET);
    unsigned char pre[12];
    if (std::fread(pre, 1, 10, f) != 10 || std::memcmp(pre, "\x93NUMPY", 6) != 0) {
        std::fclose(f);
        return "not a .npy file";
    }
    int64_t hlen, hstart;
    if (pre[6] == 1) {
        hlen = pre[8] | (pre[9] << 8);
        hstart = 10;
    } else if (pre[6] == 2 || pre[6] == 3) {
        if (std::fread(pre + 10, 1, 2, f) != 2) {
            std::fclose(f);
            return "truncated header";
        }
        hlen = static_cast<int64_t>(pre[8]) | (static_cast<int64_t>(pre[9]) << 8) |
               (static_cast<int64_t>(pre[10]) << 16) | (static_cast<int64_t>(pre[11]) << 24);
        hstart = 12;
    } else {
        std::fclose(f);
        return "unsupported .npy version";
    }
    if (hlen <= 0 || hlen > (1 << 20)) {
        std::fclose(f);
        return "bad header length";
    }
    std::string h(static_cast<size_t>(hlen), '\0');
    const size_t got = std::fread(&h[0], 1, h.size(), f);
    std::fclose(f);
    if (got != h.size()) return "truncated header";
    std::string descr = dict_value(h, "descr");
    if (descr.size() < 2 || descr.front() != '\'' || descr.back() != '\'') return "no dtype";
    out->descr = descr.substr(1, descr.size() - 2);
    if (item_size(out->descr) == 0) return "unsupported dtype " + out->descr;
    if (out->descr[0] == '>') return "big-endian data";
    const std::string fo = dict_value(h, "fortran_order");
    if (fo.find("False") == std::string::npos) return "Fortran order";
    const std::string sh = dict_value(h, "shape");
    if (sh.size() < 2 || sh.front() != '(') return "no shape";
    out->shape.clear();
    size_t p = 1;
    while (p < sh.size()) {
        while (p < sh.size() && (sh[p] == ' ' || sh[p] == ',')) ++p;
        if (p >= sh.size() || sh[p] == ')') break;
        if (sh[p] < '0' || sh[p] > '9') return "bad shape";
        int64_t v = 0;
        while (p < sh.size() && sh[p] >= '0' && sh[p] <= '9') {
            v = v * 10 + (sh[p] - '0');
            if (v > (int64_t(1) << 40)) return "shape too large";
            ++p;
        }
        out->shape.push_back(v);
    }
    // element count and bytes within 2^40 each, so the length check below
    // cannot overflow
    int64_t elems = 1;
    for (int64_t v : out->shape) {
        if (v != 0 && elems > (int64_t(1) << 40) / v) return "shape too large";
        elems *= v;
    }
    if (elems > (int64_t(1) << 40) / item_size(out->descr)) return "shape too large";
    out->data_offset = hstart + hlen;
    const int64_t need = out->data_offset + count(out->shape) * item_size(out->descr);
    if (out->file_bytes < need) return "file shorter than its shape";
    return "";
}

}  // namespace npy
}  // namespace ah

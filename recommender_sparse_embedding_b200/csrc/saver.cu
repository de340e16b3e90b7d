// saver.cu -- SafeTensors saver and loader of a table (RecIS README, Core
// architecture > Saver: sparse parameters are stored and delivered in the
// SafeTensors standard format).
//
// File layout (the SafeTensors format): an 8-byte little-endian header length
// n, n bytes of JSON header, then the tensor bytes.  The header maps each
// tensor name to {"dtype", "shape", "data_offsets": [begin, end]} (offsets
// into the byte area) and holds a "__metadata__" object of string pairs.  A
// table is saved as
//   keys    I64 [n]        the IDs, in ascending row order
//   emb     F32 [n, D]     their embedding rows
//   accum   F32 [n, D]     Adagrad accumulator      (Adagrad tables)
//   adam_m  F32 [n, D]     Adam first moment        (Adam tables)
//   adam_v  F32 [n, D]     Adam second moment       (Adam tables)
// with metadata format, dim, optimizer, step, rows and the optimiser and
// initialiser settings.  The rows stream through host memory in chunks of
// about 64 MB and land at their offsets with positioned writes, so a table
// larger than host memory can be saved.  Loading appends the file's rows to a
// table of the same dim and optimiser (keys must be new) and sets its step.
#include <fcntl.h>
#include <unistd.h>

#include <cerrno>
#include <cinttypes>
#include <cstdio>
#include <cstring>
#include <map>
#include <string>
#include <vector>

#include "internal.h"

namespace recis {
namespace {

// ---------------------------------------------------------------- JSON
// A small parser for the header: objects, arrays, strings, integers (the
// subset SafeTensors headers use; other numbers and literals are skipped).
struct JVal {
  enum Kind { kNull, kNum, kStr, kArr, kObj } kind = kNull;
  int64_t num = 0;
  std::string str;
  std::vector<JVal> arr;
  std::map<std::string, JVal> obj;
};

struct JParser {
  const char* s;
  const char* e;
  bool ok = true;
  void ws() {
    while (s < e && (*s == ' ' || *s == '\n' || *s == '\t' || *s == '\r')) ++s;
  }
  bool lit(char c) {
    ws();
    if (s < e && *s == c) {
      ++s;
      return true;
    }
    return false;
  }
  std::string string() {
    std::string out;
    if (!lit('"')) {
      ok = false;
      return out;
    }
    while (s < e && *s != '"') {
      if (*s == '\\' && s + 1 < e) {
        ++s;
        const char c = *s++;
        if (c == 'u') {  // \uXXXX: kept as '?' (names here are plain ASCII)
          s += 4;
          out.push_back('?');
        } else {
          out.push_back(c == 'n' ? '\n' : c == 't' ? '\t' : c == 'r' ? '\r' : c == 'b' ? '\b' : c == 'f' ? '\f' : c);
        }
      } else {
        out.push_back(*s++);
      }
    }
    if (s >= e) ok = false;
    ++s;
    return out;
  }
  JVal value() {
    JVal v;
    ws();
    if (s >= e) {
      ok = false;
      return v;
    }
    if (*s == '{') {
      ++s;
      v.kind = JVal::kObj;
      if (lit('}')) return v;
      do {
        std::string k = string();
        if (!ok || !lit(':')) {
          ok = false;
          return v;
        }
        v.obj[k] = value();
        if (!ok) return v;
      } while (lit(','));
      if (!lit('}')) ok = false;
    } else if (*s == '[') {
      ++s;
      v.kind = JVal::kArr;
      if (lit(']')) return v;
      do {
        v.arr.push_back(value());
        if (!ok) return v;
      } while (lit(','));
      if (!lit(']')) ok = false;
    } else if (*s == '"') {
      v.kind = JVal::kStr;
      v.str = string();
    } else if (*s == '-' || (*s >= '0' && *s <= '9')) {
      v.kind = JVal::kNum;
      bool neg = *s == '-';
      if (neg) ++s;
      int64_t x = 0;
      while (s < e && *s >= '0' && *s <= '9') x = x * 10 + (*s++ - '0');
      while (s < e && (*s == '.' || *s == 'e' || *s == 'E' || *s == '+' || *s == '-' || (*s >= '0' && *s <= '9')))
        ++s;  // fractional or exponent part: not used by the headers read here
      v.num = neg ? -x : x;
    } else {  // true / false / null
      while (s < e && *s >= 'a' && *s <= 'z') ++s;
    }
    return v;
  }
};

std::string jstr(const std::string& x) {
  std::string o = "\"";
  for (char c : x) {
    if (c == '"' || c == '\\') o.push_back('\\');
    o.push_back(c);
  }
  return o + "\"";
}

std::string fmt_double(double x) {
  char b[64];
  std::snprintf(b, sizeof(b), "%.17g", x);
  return b;
}

bool pwrite_all(int fd, const void* buf, size_t n, uint64_t off) {
  const char* p = static_cast<const char*>(buf);
  while (n > 0) {
    const ssize_t w = ::pwrite(fd, p, n, (off_t)off);
    if (w <= 0) {
      if (w < 0 && errno == EINTR) continue;
      return false;
    }
    p += w;
    n -= (size_t)w;
    off += (uint64_t)w;
  }
  return true;
}

bool pread_all(int fd, void* buf, size_t n, uint64_t off) {
  char* p = static_cast<char*>(buf);
  while (n > 0) {
    const ssize_t r = ::pread(fd, p, n, (off_t)off);
    if (r <= 0) {
      if (r < 0 && errno == EINTR) continue;
      return false;
    }
    p += r;
    n -= (size_t)r;
    off += (uint64_t)r;
  }
  return true;
}

struct Fd {
  int fd = -1;
  ~Fd() {
    if (fd >= 0) ::close(fd);
  }
};

const char* state_name(int opt, int k) {
  if (opt == RECIS_ADAGRAD) return "accum";
  return k == 0 ? "adam_m" : "adam_v";
}

}  // namespace
}  // namespace recis

using namespace recis;

extern "C" recis_status recis_table_save(recis_table_t t, const char* path, recis_stream_t stream) {
  if (!t || !path) {
    set_error("table_save: null argument");
    return RECIS_ERR_INVALID_ARG;
  }
  int64_t nrows = 0;  // rows in use: live rows and freed ones (key -1) below them
  recis_status st = table_counts(t, (cudaStream_t)stream, &nrows, nullptr);
  if (st != RECIS_OK) return st;
  const int64_t step = t->step;
  const int D = t->D, S = t->s;
  // the live rows (free rows hold key -1) in ascending row order
  std::vector<int64_t> keys((size_t)std::max<int64_t>(nrows, 1));
  if (nrows > 0) {
    const cudaError_t e = cudaMemcpy(keys.data(), (const void*)t->keys.va, sizeof(int64_t) * nrows,
                                     cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "table_save: keys");
  }
  int64_t n = 0;
  for (int64_t r = 0; r < nrows; ++r) n += keys[r] != kEmptyKey;
  // header
  const uint64_t kb = (uint64_t)n * 8, eb = (uint64_t)n * D * 4;
  std::string h = "{";
  uint64_t off = 0;
  auto tensor = [&](const std::string& name, const char* dt, const std::string& shape, uint64_t bytes) {
    h += jstr(name) + ":{\"dtype\":\"" + dt + "\",\"shape\":" + shape + ",\"data_offsets\":[" +
         std::to_string(off) + "," + std::to_string(off + bytes) + "]},";
    off += bytes;
  };
  const std::string vshape = "[" + std::to_string(n) + "," + std::to_string(D) + "]";
  tensor("keys", "I64", "[" + std::to_string(n) + "]", kb);
  tensor("emb", "F32", vshape, eb);
  for (int k = 0; k < S; ++k) tensor(state_name(t->cfg.optimizer, k), "F32", vshape, eb);
  const recis_table_config& c = t->cfg;
  h += "\"__metadata__\":{\"format\":\"recis-embedding-table\",\"dim\":" + jstr(std::to_string(D)) +
       ",\"optimizer\":" + jstr(c.optimizer == RECIS_ADAM ? "adam" : "adagrad") + ",\"step\":" +
       jstr(std::to_string(step)) + ",\"rows\":" + jstr(std::to_string(n)) + ",\"lr\":" + jstr(fmt_double(c.lr)) +
       ",\"beta1\":" + jstr(fmt_double(c.beta1)) + ",\"beta2\":" + jstr(fmt_double(c.beta2)) + ",\"eps\":" +
       jstr(fmt_double(c.eps)) + ",\"adagrad_init_acc\":" + jstr(fmt_double(c.adagrad_init_acc)) +
       ",\"init_scale\":" + jstr(fmt_double(c.init_scale)) + ",\"init_seed\":" + jstr(std::to_string(c.init_seed)) +
       "}}";
  while ((h.size() + 8) % 8 != 0) h.push_back(' ');  // the byte area starts 8-byte aligned
  Fd f;
  f.fd = ::open(path, O_WRONLY | O_CREAT | O_TRUNC, 0644);
  if (f.fd < 0) {
    set_error(std::string("table_save: cannot open ") + path + ": " + std::strerror(errno));
    return RECIS_ERR_INVALID_ARG;
  }
  const uint64_t hn = h.size();
  uint8_t len8[8];
  for (int i = 0; i < 8; ++i) len8[i] = (uint8_t)(hn >> (8 * i));
  if (!pwrite_all(f.fd, len8, 8, 0) || !pwrite_all(f.fd, h.data(), hn, 8)) {
    set_error("table_save: write failed");
    return RECIS_ERR_INVALID_ARG;
  }
  const uint64_t base = 8 + hn;
  // rows in chunks: [emb | state] rows from the device, split per tensor
  const int64_t chunk = std::max<int64_t>(1, ((int64_t)64 << 20) / (int64_t)t->row_bytes);
  std::vector<float> buf((size_t)std::min(chunk, std::max<int64_t>(nrows, 1)) * t->row_floats);
  std::vector<int64_t> ko;
  std::vector<float> eo, so[2];
  int64_t done = 0;  // live rows written so far
  for (int64_t r0 = 0; r0 < nrows; r0 += chunk) {
    const int64_t nr = std::min(chunk, nrows - r0);
    const cudaError_t e = cudaMemcpy(buf.data(), (const char*)t->rows.va + (size_t)r0 * t->row_bytes,
                                     (size_t)nr * t->row_bytes, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "table_save: rows");
    ko.clear();
    eo.clear();
    so[0].clear();
    so[1].clear();
    for (int64_t i = 0; i < nr; ++i) {
      if (keys[r0 + i] == kEmptyKey) continue;
      const float* src = buf.data() + (size_t)i * t->row_floats;
      ko.push_back(keys[r0 + i]);
      eo.insert(eo.end(), src, src + D);
      for (int k = 0; k < S; ++k) so[k].insert(so[k].end(), src + D * (1 + k), src + D * (2 + k));
    }
    const uint64_t m = ko.size();
    bool ok = pwrite_all(f.fd, ko.data(), m * 8, base + (uint64_t)done * 8) &&
              pwrite_all(f.fd, eo.data(), m * D * 4, base + kb + (uint64_t)done * D * 4);
    for (int k = 0; k < S && ok; ++k)
      ok = pwrite_all(f.fd, so[k].data(), m * D * 4, base + kb + eb * (1 + k) + (uint64_t)done * D * 4);
    if (!ok) {
      set_error("table_save: write failed");
      return RECIS_ERR_INVALID_ARG;
    }
    done += (int64_t)m;
  }
  if (::fsync(f.fd) != 0) {
    set_error("table_save: fsync failed");
    return RECIS_ERR_INVALID_ARG;
  }
  return RECIS_OK;
}

extern "C" recis_status recis_table_load(recis_table_t t, const char* path, recis_stream_t stream) {
  if (!t || !path) {
    set_error("table_load: null argument");
    return RECIS_ERR_INVALID_ARG;
  }
  Fd f;
  f.fd = ::open(path, O_RDONLY);
  if (f.fd < 0) {
    set_error(std::string("table_load: cannot open ") + path + ": " + std::strerror(errno));
    return RECIS_ERR_INVALID_ARG;
  }
  uint8_t len8[8];
  if (!pread_all(f.fd, len8, 8, 0)) {
    set_error("table_load: short file");
    return RECIS_ERR_INVALID_ARG;
  }
  uint64_t hn = 0;
  for (int i = 0; i < 8; ++i) hn |= (uint64_t)len8[i] << (8 * i);
  if (hn > ((uint64_t)1 << 30)) {
    set_error("table_load: header too large");
    return RECIS_ERR_INVALID_ARG;
  }
  std::string h(hn, ' ');
  if (!pread_all(f.fd, &h[0], hn, 8)) {
    set_error("table_load: short header");
    return RECIS_ERR_INVALID_ARG;
  }
  JParser jp{h.data(), h.data() + h.size()};
  const JVal root = jp.value();
  if (!jp.ok || root.kind != JVal::kObj) {
    set_error("table_load: malformed header");
    return RECIS_ERR_INVALID_ARG;
  }
  const int D = t->D, S = t->s;
  struct Tn {
    uint64_t begin = 0, end = 0;
    int64_t rows = -1;
  };
  auto find = [&](const char* name, const char* dt, int cols, Tn* out) -> bool {
    auto it = root.obj.find(name);
    if (it == root.obj.end() || it->second.kind != JVal::kObj) return false;
    const auto& o = it->second.obj;
    auto d = o.find("dtype"), sh = o.find("shape"), of = o.find("data_offsets");
    if (d == o.end() || sh == o.end() || of == o.end() || d->second.str != dt ||
        of->second.arr.size() != 2 || sh->second.kind != JVal::kArr)
      return false;
    const auto& s = sh->second.arr;
    if (cols == 0 ? s.size() != 1 : (s.size() != 2 || s[1].num != cols)) return false;
    out->rows = s[0].num;
    out->begin = (uint64_t)of->second.arr[0].num;
    out->end = (uint64_t)of->second.arr[1].num;
    return out->end - out->begin == (uint64_t)out->rows * (cols == 0 ? 8 : (uint64_t)cols * 4);
  };
  Tn tk, te, ts[2];
  bool ok = find("keys", "I64", 0, &tk) && find("emb", "F32", D, &te) && te.rows == tk.rows;
  for (int k = 0; k < S && ok; ++k)
    ok = find(state_name(t->cfg.optimizer, k), "F32", D, &ts[k]) && ts[k].rows == tk.rows;
  if (!ok) {
    set_error("table_load: the file does not hold keys, emb and this table's optimiser state with dim " +
              std::to_string(D));
    return RECIS_ERR_INVALID_ARG;
  }
  int64_t step = 0;
  auto md = root.obj.find("__metadata__");
  if (md != root.obj.end() && md->second.kind == JVal::kObj) {
    auto sp = md->second.obj.find("step");
    if (sp != md->second.obj.end()) step = std::strtoll(sp->second.str.c_str(), nullptr, 10);
  }
  const int64_t n = tk.rows;
  const uint64_t base = 8 + hn;
  // append in chunks through recis_table_import (keys must be new)
  const int64_t chunk = std::max<int64_t>(1, ((int64_t)32 << 20) / (int64_t)t->row_bytes);
  std::vector<int64_t> kk;
  std::vector<float> ee, ss;
  std::vector<float> sk[2];
  for (int64_t r0 = 0; r0 < n || (n == 0 && r0 == 0); r0 += chunk) {
    const int64_t nr = std::min(chunk, n - r0);
    kk.resize((size_t)std::max<int64_t>(nr, 1));
    ee.resize((size_t)std::max<int64_t>(nr, 1) * D);
    ss.resize((size_t)std::max<int64_t>(nr, 1) * D * S);
    bool rd = nr <= 0 || (pread_all(f.fd, kk.data(), (size_t)nr * 8, base + tk.begin + (uint64_t)r0 * 8) &&
                          pread_all(f.fd, ee.data(), (size_t)nr * D * 4, base + te.begin + (uint64_t)r0 * D * 4));
    for (int k = 0; k < S && rd && nr > 0; ++k) {
      sk[k].resize((size_t)nr * D);
      rd = pread_all(f.fd, sk[k].data(), (size_t)nr * D * 4, base + ts[k].begin + (uint64_t)r0 * D * 4);
    }
    if (!rd) {
      set_error("table_load: short data");
      return RECIS_ERR_INVALID_ARG;
    }
    for (int64_t i = 0; i < nr; ++i)
      for (int k = 0; k < S; ++k)
        std::memcpy(&ss[((size_t)i * S + k) * D], &sk[k][(size_t)i * D], sizeof(float) * D);
    const recis_status st = recis_table_import(t, kk.data(), ee.data(), ss.data(), std::max<int64_t>(nr, 0),
                                               step, stream);
    if (st != RECIS_OK) return st;
    if (n == 0) break;
  }
  return RECIS_OK;
}

// Checkpoint loader: a single-file safetensors checkpoint of a wav2vec2 CTC
// model (the pages' builder reads `model.safetensors` and keeps the
// checkpoint's tensor names and dtypes) packed into the float32 weight blob of
// w2v_create, host side only.
//
// File format: an 8-byte little-endian header length H, H bytes of JSON
//   {"<tensor name>": {"dtype": "F32"|"F16"|"BF16"|"F64", "shape": [...],
//                      "data_offsets": [begin, end]}, ..., "__metadata__": {...}}
// then the raw little-endian data, offsets relative to the end of the header.
//
// Names: every manifest entry is looked up under its own name, then under the
// checkpoint's module path, with or without the "wav2vec2." prefix of a CTC
// model (w2v.h lists the map).  The positional conv carries weight
// normalisation in a checkpoint (a magnitude g and a direction v); it is
// folded into the static weight g * v / ||v|| here, the norm taken over every
// axis where g has extent 1 (the pages' "pos_conv weight-norm folded into a
// static weight").
#include <cmath>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <map>
#include <memory>
#include <string>
#include <vector>

#include "w2v.h"

namespace {

struct TensorInfo {
  std::string dtype;
  std::vector<int64_t> shape;
  uint64_t begin = 0, end = 0;
};

// Minimal JSON reader for the header: objects, arrays, strings, numbers,
// true/false/null.  Only the fields above are kept.
struct Json {
  const char* p;
  const char* e;
  std::string err;

  void ws() {
    while (p < e && (*p == ' ' || *p == '\t' || *p == '\n' || *p == '\r')) ++p;
  }
  bool lit(char c) {
    ws();
    if (p < e && *p == c) {
      ++p;
      return true;
    }
    return false;
  }
  bool str(std::string* out) {
    ws();
    if (p >= e || *p != '"') return fail("string expected");
    ++p;
    out->clear();
    while (p < e && *p != '"') {
      if (*p == '\\') {
        if (++p >= e) return fail("bad escape");
        switch (*p) {
          case 'n': out->push_back('\n'); break;
          case 't': out->push_back('\t'); break;
          case 'r': out->push_back('\r'); break;
          case 'b': out->push_back('\b'); break;
          case 'f': out->push_back('\f'); break;
          case 'u': {  // keep ASCII, replace the rest (names here are ASCII)
            if (e - p < 5) return fail("bad \\u escape");
            unsigned v = 0;
            for (int i = 1; i <= 4; ++i) {
              const char c = p[i];
              v = v * 16 + (c >= '0' && c <= '9' ? c - '0' : c >= 'a' && c <= 'f' ? c - 'a' + 10 : c >= 'A' && c <= 'F' ? c - 'A' + 10 : 0);
            }
            out->push_back(v < 128 ? static_cast<char>(v) : '?');
            p += 4;
            break;
          }
          default: out->push_back(*p);
        }
        ++p;
      } else {
        out->push_back(*p++);
      }
    }
    if (p >= e) return fail("unterminated string");
    ++p;
    return true;
  }
  bool num(int64_t* out) {
    ws();
    const char* s = p;
    if (p < e && (*p == '-' || *p == '+')) ++p;
    while (p < e && ((*p >= '0' && *p <= '9') || *p == '.' || *p == 'e' || *p == 'E' || *p == '-' || *p == '+')) ++p;
    if (p == s) return fail("number expected");
    const std::string t(s, p);
    char* q = nullptr;
    const long long v = std::strtoll(t.c_str(), &q, 10);
    if (q != t.c_str() + t.size()) return fail("integer expected");
    *out = v;
    return true;
  }
  bool skip() {  // any value
    ws();
    if (p >= e) return fail("value expected");
    if (*p == '"') {
      std::string t;
      return str(&t);
    }
    if (*p == '{' || *p == '[') {
      const char close = *p == '{' ? '}' : ']';
      const bool obj = *p == '{';
      ++p;
      if (lit(close)) return true;
      for (;;) {
        if (obj) {
          std::string k;
          if (!str(&k) || !lit(':')) return fail("bad object");
        }
        if (!skip()) return false;
        if (lit(close)) return true;
        if (!lit(',')) return fail("',' expected");
      }
    }
    while (p < e && *p != ',' && *p != '}' && *p != ']' && *p != ' ' && *p != '\n') ++p;
    return true;
  }
  bool tensor(TensorInfo* t) {
    if (!lit('{')) return fail("tensor object expected");
    if (lit('}')) return true;
    for (;;) {
      std::string k;
      if (!str(&k) || !lit(':')) return fail("bad tensor entry");
      if (k == "dtype") {
        if (!str(&t->dtype)) return false;
      } else if (k == "shape" || k == "data_offsets") {
        std::vector<int64_t> v;
        if (!lit('[')) return fail("array expected");
        if (!lit(']')) {
          for (;;) {
            int64_t x = 0;
            if (!num(&x)) return false;
            v.push_back(x);
            if (lit(']')) break;
            if (!lit(',')) return fail("',' expected");
          }
        }
        if (k == "shape") {
          t->shape = v;
        } else {
          if (v.size() != 2 || v[0] < 0 || v[1] < v[0]) return fail("bad data_offsets");
          t->begin = static_cast<uint64_t>(v[0]);
          t->end = static_cast<uint64_t>(v[1]);
        }
      } else if (!skip()) {
        return false;
      }
      if (lit('}')) return true;
      if (!lit(',')) return fail("',' expected");
    }
  }
  bool header(std::map<std::string, TensorInfo>* out) {
    if (!lit('{')) return fail("header must be an object");
    if (lit('}')) return true;
    for (;;) {
      std::string k;
      if (!str(&k) || !lit(':')) return fail("bad header entry");
      if (k == "__metadata__") {
        if (!skip()) return false;
      } else {
        TensorInfo t;
        if (!tensor(&t)) return false;
        (*out)[k] = t;
      }
      if (lit('}')) return true;
      if (!lit(',')) return fail("',' expected");
    }
  }
  bool fail(const char* m) {
    if (err.empty()) err = m;
    return false;
  }
};

struct File {
  std::map<std::string, TensorInfo> tensors;
  std::vector<uint8_t> data;  // everything after the header
};

int set_err(char* err, size_t len, int code, const char* fmt, ...) {
  if (err && len) {
    va_list ap;
    va_start(ap, fmt);
    std::vsnprintf(err, len, fmt, ap);
    va_end(ap);
  }
  return code;
}

int read_file(const char* path, File* f, char* err, size_t len) {
  FILE* fp = std::fopen(path, "rb");
  if (!fp) return set_err(err, len, W2V_EINVAL, "cannot open %s", path);
  std::unique_ptr<FILE, int (*)(FILE*)> guard(fp, std::fclose);
  uint8_t hb[8];
  if (std::fread(hb, 1, 8, fp) != 8) return set_err(err, len, W2V_EINVAL, "%s: no header length", path);
  uint64_t hl = 0;
  for (int i = 7; i >= 0; --i) hl = (hl << 8) | hb[i];
  if (hl == 0 || hl > (100u << 20)) return set_err(err, len, W2V_EINVAL, "%s: header length %llu out of range", path,
                                                 static_cast<unsigned long long>(hl));
  std::string hdr(hl, '\0');
  if (std::fread(&hdr[0], 1, hl, fp) != hl) return set_err(err, len, W2V_EINVAL, "%s: truncated header", path);
  Json j{hdr.data(), hdr.data() + hdr.size(), {}};
  if (!j.header(&f->tensors)) return set_err(err, len, W2V_EINVAL, "%s: bad header (%s)", path, j.err.c_str());
  if (std::fseek(fp, 0, SEEK_END) != 0) return set_err(err, len, W2V_EINVAL, "%s: cannot seek", path);
  const long total = std::ftell(fp);
  if (total < 0 || static_cast<uint64_t>(total) < 8 + hl) return set_err(err, len, W2V_EINVAL, "%s: bad size", path);
  const uint64_t n = static_cast<uint64_t>(total) - 8 - hl;
  f->data.resize(n);
  if (std::fseek(fp, static_cast<long>(8 + hl), SEEK_SET) != 0 || (n && std::fread(f->data.data(), 1, n, fp) != n))
    return set_err(err, len, W2V_EINVAL, "%s: cannot read data", path);
  for (auto& kv : f->tensors)
    if (kv.second.end > n)
      return set_err(err, len, W2V_EINVAL, "%s: tensor %s lies past the end of the file", path, kv.first.c_str());
  return W2V_OK;
}

int elem_size(const std::string& dt) {
  if (dt == "F32") return 4;
  if (dt == "F16" || dt == "BF16") return 2;
  if (dt == "F64") return 8;
  return 0;
}

float half_to_float(uint16_t h) {
  const uint32_t s = (h >> 15) & 1u, ex = (h >> 10) & 31u, m = h & 1023u;
  float v;
  if (ex == 0) v = std::ldexp(static_cast<float>(m), -24);
  else if (ex == 31) v = m ? NAN : INFINITY;
  else v = std::ldexp(static_cast<float>(m | 1024u), static_cast<int>(ex) - 25);
  return s ? -v : v;
}

// The tensor as float64 values (fp16 / bf16 / fp32 are exact in float64).
std::vector<double> to_f64(const File& f, const TensorInfo& t) {
  const size_t es = static_cast<size_t>(elem_size(t.dtype));
  const size_t n = (t.end - t.begin) / es;
  std::vector<double> v(n);
  const uint8_t* p = f.data.data() + t.begin;
  for (size_t i = 0; i < n; ++i) {
    if (t.dtype == "F32") {
      float x;
      std::memcpy(&x, p + 4 * i, 4);
      v[i] = x;
    } else if (t.dtype == "F64") {
      std::memcpy(&v[i], p + 8 * i, 8);
    } else {
      uint16_t h;
      std::memcpy(&h, p + 2 * i, 2);
      if (t.dtype == "F16") {
        v[i] = half_to_float(h);
      } else {
        const uint32_t b = static_cast<uint32_t>(h) << 16;
        float x;
        std::memcpy(&x, &b, 4);
        v[i] = x;
      }
    }
  }
  return v;
}

// Checkpoint module paths of a manifest name (without the model prefix).
std::vector<std::string> checkpoint_names(const std::string& n) {
  std::vector<std::string> out;
  auto starts = [&](const char* s) { return n.compare(0, std::strlen(s), s) == 0; };
  auto tail = [&](size_t pos) { return n.substr(pos); };
  if (starts("conv") && n.size() > 5 && n[5] == '.') {
    const std::string i(1, n[4]);
    const std::string rest = tail(6);  // weight, bias, norm.weight, norm.bias
    if (rest.compare(0, 5, "norm.") == 0)
      out.push_back("feature_extractor.conv_layers." + i + ".layer_norm." + rest.substr(5));
    else
      out.push_back("feature_extractor.conv_layers." + i + ".conv." + rest);
  } else if (starts("fp.norm.")) {
    out.push_back("feature_projection.layer_norm." + tail(8));
  } else if (starts("fp.proj.")) {
    out.push_back("feature_projection.projection." + tail(8));
  } else if (starts("pos_conv.")) {
    out.push_back("encoder.pos_conv_embed.conv." + tail(9));
  } else if (starts("enc.norm.")) {
    out.push_back("encoder.layer_norm." + tail(9));
  } else if (starts("layers.")) {
    const size_t dot = n.find('.', 7);
    const std::string l = n.substr(7, dot - 7), rest = n.substr(dot + 1);
    const std::string pre = "encoder.layers." + l + ".";
    const char* attn[4][2] = {{"attn.q.", "attention.q_proj."},
                              {"attn.k.", "attention.k_proj."},
                              {"attn.v.", "attention.v_proj."},
                              {"attn.out.", "attention.out_proj."}};
    for (auto& a : attn)
      if (rest.compare(0, std::strlen(a[0]), a[0]) == 0) out.push_back(pre + a[1] + rest.substr(std::strlen(a[0])));
    if (rest.compare(0, 10, "attn_norm.") == 0) out.push_back(pre + "layer_norm." + rest.substr(10));
    if (rest.compare(0, 7, "ffn.in.") == 0) out.push_back(pre + "feed_forward.intermediate_dense." + rest.substr(7));
    if (rest.compare(0, 8, "ffn.out.") == 0) out.push_back(pre + "feed_forward.output_dense." + rest.substr(8));
    if (rest.compare(0, 9, "ffn_norm.") == 0) out.push_back(pre + "final_layer_norm." + rest.substr(9));
  } else if (starts("lm_head.")) {
    out.push_back(n);
  }
  return out;
}

const TensorInfo* find(const File& f, const std::string& name, std::string* found) {
  auto it = f.tensors.find(name);
  if (it != f.tensors.end()) {
    *found = name;
    return &it->second;
  }
  return nullptr;
}

// First of: the manifest name, then each checkpoint path with and without the
// CTC model's "wav2vec2." prefix, each with the suffix `suffix` replacing the
// last component when given (weight-norm parts).
const TensorInfo* lookup(const File& f, const std::string& mname, const std::string& suffix, std::string* found) {
  std::vector<std::string> cands;
  auto with_suffix = [&](const std::string& s) {
    if (suffix.empty()) return s;
    const size_t dot = s.rfind('.');
    return s.substr(0, dot + 1) + suffix;
  };
  cands.push_back(with_suffix(mname));
  for (const std::string& c : checkpoint_names(mname)) {
    cands.push_back(with_suffix(c));
    cands.push_back("wav2vec2." + with_suffix(c));
  }
  for (const std::string& c : cands)
    if (const TensorInfo* t = find(f, c, found)) return t;
  return nullptr;
}

bool same_shape(const TensorInfo& t, int ndim, const int64_t* shape) {
  if (static_cast<int>(t.shape.size()) != ndim) return false;
  for (int i = 0; i < ndim; ++i)
    if (t.shape[i] != shape[i]) return false;
  return true;
}

std::string shape_str(const std::vector<int64_t>& s) {
  std::string r = "[";
  for (size_t i = 0; i < s.size(); ++i) r += (i ? ", " : "") + std::to_string(s[i]);
  return r + "]";
}

int checked_tensor(const File& f, const TensorInfo& t, const std::string& name, char* err, size_t len) {
  const int es = elem_size(t.dtype);
  if (!es) return set_err(err, len, W2V_EINVAL, "%s: unsupported dtype %s", name.c_str(), t.dtype.c_str());
  uint64_t cnt = 1;
  for (int64_t d : t.shape) {
    if (d < 0) return set_err(err, len, W2V_EINVAL, "%s: negative extent", name.c_str());
    cnt *= static_cast<uint64_t>(d);
  }
  if (cnt * es != t.end - t.begin)
    return set_err(err, len, W2V_EINVAL, "%s: data size does not match its shape", name.c_str());
  (void)f;
  return W2V_OK;
}

// Weight normalisation folded: w = g * v / ||v||, the norm over every axis
// where g has extent 1 (one norm per index of g's other axes).
int fold_weight_norm(const File& f, const TensorInfo& g, const TensorInfo& v, const std::string& name, float* out,
                     char* err, size_t len) {
  if (g.shape.size() != v.shape.size())
    return set_err(err, len, W2V_ESHAPE, "%s: weight-norm g %s and v %s differ in rank", name.c_str(),
                   shape_str(g.shape).c_str(), shape_str(v.shape).c_str());
  const int nd = static_cast<int>(v.shape.size());
  for (int i = 0; i < nd; ++i)
    if (g.shape[i] != 1 && g.shape[i] != v.shape[i])
      return set_err(err, len, W2V_ESHAPE, "%s: weight-norm g %s does not broadcast over v %s", name.c_str(),
                     shape_str(g.shape).c_str(), shape_str(v.shape).c_str());
  const std::vector<double> gv = to_f64(f, g), vv = to_f64(f, v);
  const size_t n = vv.size();
  // index of g for each element of v
  std::vector<size_t> gi(n);
  std::vector<int64_t> idx(nd, 0);
  for (size_t e = 0; e < n; ++e) {
    size_t k = 0;
    for (int a = 0; a < nd; ++a) k = k * static_cast<size_t>(g.shape[a]) + (g.shape[a] == 1 ? 0 : idx[a]);
    gi[e] = k;
    for (int a = nd - 1; a >= 0; --a) {
      if (++idx[a] < v.shape[a]) break;
      idx[a] = 0;
    }
  }
  std::vector<double> ss(gv.size(), 0.0);
  for (size_t e = 0; e < n; ++e) ss[gi[e]] += vv[e] * vv[e];
  for (size_t e = 0; e < n; ++e) {
    const double nrm = std::sqrt(ss[gi[e]]);
    out[e] = static_cast<float>(nrm > 0.0 ? gv[gi[e]] * vv[e] / nrm : 0.0);
  }
  return W2V_OK;
}

}  // namespace

extern "C" int w2v_pack_safetensors(const char* path, const w2v_config* cfg, float* blob, size_t n_floats, char* err,
                                    size_t err_len) {
  if (err && err_len) err[0] = '\0';
  if (!path || !cfg || !blob) return set_err(err, err_len, W2V_EINVAL, "null argument");
  const size_t total = w2v_weight_count(cfg);
  if (total == 0) return set_err(err, err_len, W2V_EINVAL, "invalid config");
  if (n_floats != total)
    return set_err(err, err_len, W2V_ESHAPE, "blob holds %zu floats, the config needs %zu", n_floats, total);
  File f;
  const int rc = read_file(path, &f, err, err_len);
  if (rc != W2V_OK) return rc;
  const int ne = w2v_weight_num_entries(cfg);
  for (int i = 0; i < ne; ++i) {
    char nm[128];
    int ndim = 0;
    int64_t shape[3] = {0, 0, 0};
    size_t off = 0;
    if (w2v_weight_entry(cfg, i, nm, sizeof nm, &ndim, shape, &off) != W2V_OK)
      return set_err(err, err_len, W2V_EINVAL, "manifest entry %d", i);
    const std::string mname(nm);
    size_t cnt = 1;
    for (int a = 0; a < ndim; ++a) cnt *= static_cast<size_t>(shape[a]);
    std::string found;
    const TensorInfo* t = lookup(f, mname, "", &found);
    if (!t && mname == "pos_conv.weight") {
      // weight normalisation: (weight_g, weight_v), or PyTorch's
      // parametrization (original0 = g, original1 = v)
      std::string fg, fv;
      const TensorInfo* g = lookup(f, mname, "weight_g", &fg);
      const TensorInfo* v = lookup(f, mname, "weight_v", &fv);
      if (!g || !v) {
        g = lookup(f, mname, "parametrizations.weight.original0", &fg);
        v = lookup(f, mname, "parametrizations.weight.original1", &fv);
      }
      if (g && v) {
        int r = checked_tensor(f, *g, fg, err, err_len);
        if (r == W2V_OK) r = checked_tensor(f, *v, fv, err, err_len);
        if (r != W2V_OK) return r;
        if (!same_shape(*v, ndim, shape))
          return set_err(err, err_len, W2V_ESHAPE, "%s has shape %s, %s needs [%lld, %lld, %lld]", fv.c_str(),
                         shape_str(v->shape).c_str(), nm, static_cast<long long>(shape[0]),
                         static_cast<long long>(shape[1]), static_cast<long long>(shape[2]));
        r = fold_weight_norm(f, *g, *v, fv, blob + off, err, err_len);
        if (r != W2V_OK) return r;
        continue;
      }
    }
    if (!t) return set_err(err, err_len, W2V_EINVAL, "tensor for %s not found in %s", nm, path);
    int r = checked_tensor(f, *t, found, err, err_len);
    if (r != W2V_OK) return r;
    if (!same_shape(*t, ndim, shape)) {
      std::vector<int64_t> want(shape, shape + ndim);
      return set_err(err, err_len, W2V_ESHAPE, "%s has shape %s, %s needs %s", found.c_str(),
                     shape_str(t->shape).c_str(), nm, shape_str(want).c_str());
    }
    const std::vector<double> v = to_f64(f, *t);
    for (size_t k = 0; k < cnt; ++k) blob[off + k] = static_cast<float>(v[k]);
  }
  return W2V_OK;
}

extern "C" int w2v_create_from_safetensors(const char* path, const w2v_config* cfg, w2v_model** out, char* err,
                                           size_t err_len) {
  if (!out) return set_err(err, err_len, W2V_EINVAL, "null argument");
  *out = nullptr;
  const size_t total = cfg ? w2v_weight_count(cfg) : 0;
  if (!total) return set_err(err, err_len, W2V_EINVAL, "invalid config");
  std::vector<float> blob(total);
  const int rc = w2v_pack_safetensors(path, cfg, blob.data(), total, err, err_len);
  if (rc != W2V_OK) return rc;
  const int rc2 = w2v_create(cfg, blob.data(), total, out);
  if (rc2 != W2V_OK) set_err(err, err_len, rc2, "w2v_create failed (code %d)", rc2);
  return rc2;
}

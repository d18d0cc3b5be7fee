// Static scale map: the per-layer {q, k, v} values of the vLLM docs page
// "FP8 ViT encoder attention" (scale file format section), read from and
// written to JSON text on the host, and the save-margin multiply.
//
// The file is one JSON object whose keys are layer names and whose values
// are objects holding the three numbers under "q", "k", "v" (or the
// aliases "q_scale", "k_scale", "v_scale"; the short name wins when both
// appear; other keys are ignored).  Numbers are read as doubles and rounded
// once to fp32.  Host code only: no CUDA calls.
#include <cerrno>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>

#include "fp8attn.h"

namespace {

struct Parser {
  const char* p;
  const char* end;

  void ws() {
    while (p < end && (*p == ' ' || *p == '\t' || *p == '\n' || *p == '\r')) ++p;
  }
  bool eat(char c) {
    ws();
    if (p < end && *p == c) {
      ++p;
      return true;
    }
    return false;
  }
  // A JSON string (escapes \" \\ \/ \b \f \n \r \t and \u00XX for ASCII).
  bool string(std::string* out) {
    ws();
    if (p >= end || *p != '"') return false;
    ++p;
    out->clear();
    while (p < end && *p != '"') {
      char c = *p++;
      if (static_cast<unsigned char>(c) < 0x20) return false;
      if (c != '\\') {
        out->push_back(c);
        continue;
      }
      if (p >= end) return false;
      const char e = *p++;
      switch (e) {
        case '"': out->push_back('"'); break;
        case '\\': out->push_back('\\'); break;
        case '/': out->push_back('/'); break;
        case 'b': out->push_back('\b'); break;
        case 'f': out->push_back('\f'); break;
        case 'n': out->push_back('\n'); break;
        case 'r': out->push_back('\r'); break;
        case 't': out->push_back('\t'); break;
        case 'u': {
          if (end - p < 4) return false;
          unsigned v = 0;
          for (int i = 0; i < 4; ++i) {
            const char h = *p++;
            v <<= 4;
            if (h >= '0' && h <= '9') v |= static_cast<unsigned>(h - '0');
            else if (h >= 'a' && h <= 'f') v |= static_cast<unsigned>(h - 'a' + 10);
            else if (h >= 'A' && h <= 'F') v |= static_cast<unsigned>(h - 'A' + 10);
            else return false;
          }
          if (v == 0 || v > 0x7F) return false;   // ASCII names only
          out->push_back(static_cast<char>(v));
          break;
        }
        default: return false;
      }
    }
    if (p >= end) return false;
    ++p;   // closing quote
    return true;
  }
  // A JSON number, as strtod reads it (the JSON grammar is a subset).
  bool number(double* v) {
    ws();
    if (p >= end) return false;
    const char* s = p;
    if (*s == '-') ++s;
    if (s >= end || !(*s >= '0' && *s <= '9')) return false;
    char buf[64];
    size_t n = 0;
    const char* q = p;
    while (q < end && n + 1 < sizeof(buf) &&
           (std::strchr("+-0123456789.eE", *q) != nullptr))
      buf[n++] = *q++;
    buf[n] = '\0';
    char* stop = nullptr;
    errno = 0;
    const double d = std::strtod(buf, &stop);
    if (stop == buf || errno == ERANGE) return false;
    p += (stop - buf);
    *v = d;
    return true;
  }
  // Skip any JSON value (for keys the map does not use).
  bool skip() {
    ws();
    if (p >= end) return false;
    if (*p == '"') {
      std::string s;
      return string(&s);
    }
    if (*p == '{' || *p == '[') {
      const char close = *p == '{' ? '}' : ']';
      const bool obj = *p == '{';
      ++p;
      if (eat(close)) return true;
      for (;;) {
        if (obj) {
          std::string k;
          if (!string(&k) || !eat(':')) return false;
        }
        if (!skip()) return false;
        if (eat(close)) return true;
        if (!eat(',')) return false;
      }
    }
    for (const char* lit : {"true", "false", "null"}) {
      const size_t n = std::strlen(lit);
      if (static_cast<size_t>(end - p) >= n && std::strncmp(p, lit, n) == 0) {
        p += n;
        return true;
      }
    }
    double d;
    return number(&d);
  }
};

bool margin_ok(float m) { return std::isfinite(m) && m > 0.0f; }

void append_escaped(std::string* out, const char* s) {
  out->push_back('"');
  for (; *s; ++s) {
    const unsigned char c = static_cast<unsigned char>(*s);
    if (c == '"' || c == '\\') {
      out->push_back('\\');
      out->push_back(static_cast<char>(c));
    } else if (c < 0x20) {
      char b[8];
      std::snprintf(b, sizeof(b), "\\u%04x", c);
      out->append(b);
    } else {
      out->push_back(static_cast<char>(c));
    }
  }
  out->push_back('"');
}

// Shortest decimal text that reads back as the same fp32 value.
void append_float(std::string* out, float v) {
  char b[48];
  for (int digits = 6; digits <= 9; ++digits) {
    std::snprintf(b, sizeof(b), "%.*g", digits, static_cast<double>(v));
    if (static_cast<float>(std::strtod(b, nullptr)) == v) break;
  }
  // keep it a JSON number with a fraction or exponent ("224" -> "224.0")
  if (!std::strpbrk(b, ".eEn")) std::strncat(b, ".0", sizeof(b) - std::strlen(b) - 1);
  out->append(b);
}

}  // namespace

extern "C" {

fp8attn_status fp8attn_apply_margin(const float* h_in, int64_t n, float margin, float* h_out) {
  if (n < 0 || (n > 0 && (!h_in || !h_out)) || !margin_ok(margin)) return FP8ATTN_ERR_INVALID;
  for (int64_t i = 0; i < n; ++i) h_out[i] = h_in[i] * margin;   // one fp32 rounding
  return FP8ATTN_OK;
}

fp8attn_status fp8attn_scale_map_parse(const char* json_text, size_t text_len, float margin,
                                       int max_layers, char* names_out, float* values_out,
                                       int* n_layers_out) {
  if (!json_text || !n_layers_out || max_layers < 0 || !margin_ok(margin) ||
      (max_layers > 0 && (!names_out || !values_out)))
    return FP8ATTN_ERR_INVALID;
  *n_layers_out = 0;
  Parser ps{json_text, json_text + text_len};
  if (!ps.eat('{')) return FP8ATTN_ERR_INVALID;
  int n = 0;
  if (!ps.eat('}')) {
    for (;;) {
      std::string name;
      if (!ps.string(&name) || name.size() + 1 > FP8ATTN_SCALE_NAME_MAX || !ps.eat(':') ||
          !ps.eat('{'))
        return FP8ATTN_ERR_INVALID;
      // per tensor: the value under the short key, else under the alias
      double val[3][2];
      bool have[3][2] = {{false, false}, {false, false}, {false, false}};
      if (!ps.eat('}')) {
        for (;;) {
          std::string key;
          if (!ps.string(&key) || !ps.eat(':')) return FP8ATTN_ERR_INVALID;
          int t = -1, alias = 0;
          static const char* const shortk[3] = {"q", "k", "v"};
          static const char* const longk[3] = {"q_scale", "k_scale", "v_scale"};
          for (int i = 0; i < 3; ++i) {
            if (key == shortk[i]) t = i;
            if (key == longk[i]) { t = i; alias = 1; }
          }
          if (t >= 0) {
            double d;
            if (!ps.number(&d)) return FP8ATTN_ERR_INVALID;
            val[t][alias] = d;
            have[t][alias] = true;
          } else if (!ps.skip()) {
            return FP8ATTN_ERR_INVALID;
          }
          if (ps.eat('}')) break;
          if (!ps.eat(',')) return FP8ATTN_ERR_INVALID;
        }
      }
      if (n >= max_layers) return FP8ATTN_ERR_INVALID;   // more layers than the caller's room
      for (int t = 0; t < 3; ++t) {
        if (!have[t][0] && !have[t][1]) return FP8ATTN_ERR_INVALID;
        const float stored = static_cast<float>(have[t][0] ? val[t][0] : val[t][1]);
        values_out[3 * n + t] = stored * margin;   // one fp32 rounding (exact for 1)
      }
      std::memcpy(names_out + static_cast<size_t>(n) * FP8ATTN_SCALE_NAME_MAX, name.c_str(),
                  name.size() + 1);
      ++n;
      if (ps.eat('}')) break;
      if (!ps.eat(',')) return FP8ATTN_ERR_INVALID;
    }
  }
  ps.ws();
  if (ps.p != ps.end) return FP8ATTN_ERR_INVALID;   // trailing text
  *n_layers_out = n;
  return FP8ATTN_OK;
}

fp8attn_status fp8attn_scale_map_format(int n_layers, const char* names, const float* values,
                                        char* buf, size_t buf_size, size_t* written) {
  if (n_layers < 0 || !written || (n_layers > 0 && (!names || !values))) return FP8ATTN_ERR_INVALID;
  std::string out = "{";
  for (int l = 0; l < n_layers; ++l) {
    const char* name = names + static_cast<size_t>(l) * FP8ATTN_SCALE_NAME_MAX;
    if (!std::memchr(name, '\0', FP8ATTN_SCALE_NAME_MAX)) return FP8ATTN_ERR_INVALID;
    out.append(l ? ",\n  " : "\n  ");
    append_escaped(&out, name);
    out.append(": {");
    static const char* const keys[3] = {"\"q\": ", "\"k\": ", "\"v\": "};
    for (int t = 0; t < 3; ++t) {
      const float v = values[3 * l + t];
      if (!std::isfinite(v)) return FP8ATTN_ERR_INVALID;
      out.append(t ? ", " : "");
      out.append(keys[t]);
      append_float(&out, v);
    }
    out.append("}");
  }
  out.append(n_layers ? "\n}\n" : "}\n");
  *written = out.size() + 1;
  if (!buf || buf_size < out.size() + 1) return FP8ATTN_ERR_INVALID;   // *written = room needed
  std::memcpy(buf, out.c_str(), out.size() + 1);
  return FP8ATTN_OK;
}

}  // extern "C"

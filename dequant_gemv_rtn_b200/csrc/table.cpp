// table.cpp -- per-module format table for selective precision.
//
// The RTN page ("Is (Selective) Round-To-Nearest Quantization All You Need?",
// English abstract) raises the data-precision format of selected layers and
// modules; the layer bit-width page ("A Method for Layer Bit-Width Allocation
// in LLM Quantization", English abstract) chooses precision per block of
// layers (first/last groups).  The table holds ordered (pattern -> format,
// group) rules; the first rule whose pattern matches a module name wins,
// otherwise the default applies.  Patterns: '*' any run, '?' one character.
#include <cstdlib>
#include <new>
#include <cstring>
#include <string>
#include <vector>
#include "qnt.h"

struct qnt_table {
  int default_fmt;
  int default_group;
  struct Rule {
    std::string pattern;
    int fmt;
    int group;
  };
  std::vector<Rule> rules;
};

namespace {

bool valid_fmt(int f) { return f >= QNT_INT4_ASYM && f <= QNT_FP16; }

bool valid_group(int f, int g) {
  if (f == QNT_INT8_PERCHAN || f == QNT_FP16) return true;  // group is K, resolved per matrix
  return g == 32 || g == 64 || g == 128;
}

// Glob match with '*' and '?', iterative with single backtrack point.
bool glob(const char* p, const char* s) {
  const char* star = nullptr;
  const char* back = nullptr;
  while (*s) {
    if (*p == '?' || (*p && *p == *s)) { ++p; ++s; continue; }
    if (*p == '*') { star = p++; back = s; continue; }
    if (star) { p = star + 1; s = ++back; continue; }
    return false;
  }
  while (*p == '*') ++p;
  return *p == 0;
}

}  // namespace

extern "C" {

qnt_table* qnt_table_create(int default_fmt, int default_group) {
  if (!valid_fmt(default_fmt) || !valid_group(default_fmt, default_group)) return nullptr;
  qnt_table* t = new (std::nothrow) qnt_table;
  if (!t) return nullptr;
  t->default_fmt = default_fmt;
  t->default_group = default_group;
  return t;
}

int qnt_table_set(qnt_table* t, const char* module_pattern, int fmt, int group) {
  if (!t || !module_pattern || !valid_fmt(fmt)) return QNT_ERR_ARG;
  if (!valid_group(fmt, group)) return QNT_ERR_SHAPE;
  t->rules.push_back({std::string(module_pattern), fmt, group});
  return QNT_OK;
}

int qnt_table_lookup(const qnt_table* t, const char* module_name, int* fmt, int* group) {
  if (!t || !module_name || !fmt || !group) return QNT_ERR_ARG;
  for (const auto& r : t->rules) {
    if (glob(r.pattern.c_str(), module_name)) {
      *fmt = r.fmt;
      *group = r.group;
      return QNT_OK;
    }
  }
  *fmt = t->default_fmt;
  *group = t->default_group;
  return QNT_OK;
}

int qnt_table_size(const qnt_table* t) { return t ? (int)t->rules.size() : -1; }

void qnt_table_destroy(qnt_table* t) { delete t; }

}  // extern "C"

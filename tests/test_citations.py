"""Every oracle function and every entry point of the C ABI names the passage of the pages
it follows (no GPU). An oracle function's comment cites a page (walkthrough, digest,
chooseai or tutorial) or states a format definition; a header section cites a page, or
says that it is not part of the layer or method (the measurement helper, the entry point
without a workspace)."""

import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PAGE = r"walkthrough|digest|chooseai|tutorial"


def _comment_above(lines, i):
    block = []
    j = i - 1
    while j >= 0 and (lines[j].lstrip().startswith("//") or not lines[j].strip()):
        block.append(lines[j])
        j -= 1
    return " ".join(reversed(block))


def test_every_oracle_function_cites_its_passage():
    with open(os.path.join(ROOT, "oracle", "csa_oracle.cpp"), encoding="utf-8") as f:
        lines = f.read().split("\n")
    missing, seen = [], 0
    for i, line in enumerate(lines):
        m = re.match(r"^[a-z][\w\s\*]* (or_\w+)\(", line)
        if not m:
            continue
        seen += 1
        text = _comment_above(lines, i)
        if not re.search(PAGE + r"|IEEE|OCP|OFP8|MX format", text):
            missing.append(m.group(1))
    assert seen >= 20
    assert missing == [], f"oracle functions without a cited passage: {missing}"


def test_every_abi_section_cites_its_passage():
    with open(os.path.join(ROOT, "include", "csa.h"), encoding="utf-8") as f:
        text = f.read()
    sections = text.split("/* " + "-" * 84)[1:]
    assert len(sections) >= 10
    missing = []
    for sec in sections:
        names = re.findall(r"^\w[\w\s\*]*\b((?:csa|hca)_\w+)\(", sec, re.M)
        if not names:
            continue
        if not (re.search(PAGE, sec) or re.search(r"not part of the (layer|method)", sec)):
            missing.append(names)
    assert missing == [], f"entry points without a cited passage: {missing}"
